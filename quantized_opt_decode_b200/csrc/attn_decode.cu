// Decode attention over the KV cache: for each (sequence, head),
//   o = softmax(q K^T / sqrt(d)) V  over the cached slots 0..len-1,
// the decode equation t_out = softmax(t_Q x_K^T / sqrt(.)) x_V W_O + t of the
// FlexGen walk-through (section "P/D阶段计算") in the per-head form of the
// survey notes' eq. (2), with K and V stored in the group-wise 4-bit format of
// "FlexGen研究学术报告" section 三(C) (or fp16).
//
// One CTA per (head, sequence); 4 warps; in each warp 8 tokens are in flight,
// 4 lanes per token, each lane owning d/4 contiguous dimensions (for d = 128:
// one 16-byte load of 32 codes, all inside one 64-element group).  Codes are
// dequantized in registers without materialising x_hat:
//   q . x_hat = scale * sum_e q_e code_e + min * sum_e q_e   (per group)
//   sum_t p_t x_hat_t = sum_t (p_t scale_t) code_t + sum_t p_t min_t,
// which is the dequantized value code * scale + min before its fp16 rounding.
// Pass 1 writes the scores to shared memory and finds their maximum, pass 2
// exponentiates, pass 3 streams V.  K and V are each read once.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace flexq {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ float block_reduce(float v, float* red, bool is_max) {
  v = is_max ? warp_max(v) : warp_sum(v);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kThreads / 32; ++i) r = is_max ? fmaxf(r, red[i]) : r + red[i];
  return r;
}

// Loads this lane's d/4 elements of one cached row as fp32 "codes" (4-bit) or
// values (16-bit).
template <int D, int KV_BITS>
__device__ __forceinline__ void load_row_part(const void* base, size_t slot, int c, float (&x)[D / 4]) {
  constexpr int DPL = D / 4;
  if constexpr (KV_BITS == 4) {
    const uint8_t* p = static_cast<const uint8_t*>(base) + slot * (D / 2) + c * (DPL / 2);
    uint32_t w[DPL / 8];
    if constexpr (DPL == 32) {
      const uint4 u = *reinterpret_cast<const uint4*>(p);
      w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
    } else {
      const uint2 u = *reinterpret_cast<const uint2*>(p);
      w[0] = u.x; w[1] = u.y;
    }
#pragma unroll
    for (int j = 0; j < DPL / 8; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) x[j * 8 + e] = static_cast<float>((w[j] >> (4 * e)) & 0xF);
  } else {
    const __half* p = static_cast<const __half*>(base) + slot * D + c * DPL;
#pragma unroll
    for (int j = 0; j < DPL / 8; ++j) {
      const uint4 u = reinterpret_cast<const uint4*>(p)[j];
      const __half2* h2 = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h2[e]);
        x[j * 8 + 2 * e] = f.x;
        x[j * 8 + 2 * e + 1] = f.y;
      }
    }
  }
}

template <int D, int KV_BITS>
__global__ void __launch_bounds__(kThreads) attn_decode_kernel(const __half* __restrict__ q, int ldq,
                                                               KvView kv, int heads, int len,
                                                               __half* __restrict__ out, int ldo,
                                                               float inv_sqrt_d) {
  constexpr int DPL = D / 4;
  extern __shared__ float sc[];
  __shared__ float red[kThreads / 32];
  __shared__ float part[kThreads / 32][D + 4];
  const int j = blockIdx.x, i = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = lane & 3;
  const int g = (c * DPL) / 64;  // group of this lane's dimensions
  const size_t row0 = (static_cast<size_t>(i) * heads + j) * kv.max_len;

  float qf[DPL];
  const __half* qp = q + static_cast<size_t>(i) * ldq + j * D + c * DPL;
#pragma unroll
  for (int e = 0; e < DPL; e += 2) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(qp + e));
    qf[e] = f.x;
    qf[e + 1] = f.y;
  }
  float qsum = 0.f;
#pragma unroll
  for (int e = 0; e < DPL; ++e) qsum += qf[e];

  // pass 1: scores
  float mx = -INFINITY;
  for (int base = warp * 8; base < len; base += kThreads / 4) {
    const int t = base + (lane >> 2);
    const bool valid = t < len;
    float partial = 0.f;
    if (valid) {
      float x[DPL];
      load_row_part<D, KV_BITS>(kv.k, row0 + t, c, x);
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) dot = fmaf(qf[e], x[e], dot);
      if constexpr (KV_BITS == 4) {
        const __half2 ms = static_cast<const __half2*>(kv.k_meta)[(row0 + t) * (D / 64) + g];
        const float2 f = __half22float2(ms);  // (min, scale)
        partial = f.y * dot + f.x * qsum;
      } else {
        partial = dot;
      }
    }
    partial += __shfl_xor_sync(0xffffffffu, partial, 1);
    partial += __shfl_xor_sync(0xffffffffu, partial, 2);
    if (valid) {
      const float s = partial * inv_sqrt_d;
      if (c == 0) sc[t] = s;
      mx = fmaxf(mx, s);
    }
  }
  const float M = block_reduce(mx, red, true);

  // pass 2: exponentials (scores were written before the reduction's barrier)
  float sum = 0.f;
  for (int t = threadIdx.x; t < len; t += kThreads) {
    const float p = __expf(sc[t] - M);
    sc[t] = p;
    sum += p;
  }
  const float S = block_reduce(sum, red, false);

  // pass 3: weighted sum of V
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  float am = 0.f;
  for (int base = warp * 8; base < len; base += kThreads / 4) {
    const int t = base + (lane >> 2);
    if (t < len) {
      const float p = sc[t];
      float x[DPL];
      load_row_part<D, KV_BITS>(kv.v, row0 + t, c, x);
      float w = p;
      if constexpr (KV_BITS == 4) {
        const float2 f = __half22float2(static_cast<const __half2*>(kv.v_meta)[(row0 + t) * (D / 64) + g]);
        w = p * f.y;
        am = fmaf(p, f.x, am);
      }
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(w, x[e], acc[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    float v = acc[e] + am;
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    acc[e] = v;
  }
  if (lane < 4) {
#pragma unroll
    for (int e = 0; e < DPL; ++e) part[warp][c * DPL + e] = acc[e];
  }
  __syncthreads();
  const float invS = 1.0f / S;
  for (int e = threadIdx.x; e < D; e += kThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) v += part[w][e];
    out[static_cast<size_t>(i) * ldo + j * D + e] = __float2half_rn(v * invS);
  }
}

template <int D, int KV_BITS>
cudaError_t launch_one(const __half* q, int ldq, const KvView& kv, int b, int heads, int len,
                       __half* out, int ldo, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(len) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(attn_decode_kernel<D, KV_BITS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(heads, b);
  attn_decode_kernel<D, KV_BITS><<<grid, kThreads, smem, s>>>(q, ldq, kv, heads, len, out, ldo,
                                                              1.0f / sqrtf(static_cast<float>(D)));
  return launched();
}

}  // namespace

cudaError_t launch_attn_decode(const __half* q, int ldq, const KvView& kv, int b, int heads, int d,
                               int kv_bits, int len, __half* out, int ldo, cudaStream_t s) {
  if (b == 0) return cudaSuccess;
  if (d == 128)
    return kv_bits == 4 ? launch_one<128, 4>(q, ldq, kv, b, heads, len, out, ldo, s)
                        : launch_one<128, 16>(q, ldq, kv, b, heads, len, out, ldo, s);
  return kv_bits == 4 ? launch_one<64, 4>(q, ldq, kv, b, heads, len, out, ldo, s)
                      : launch_one<64, 16>(q, ldq, kv, b, heads, len, out, ldo, s);
}

}  // namespace flexq

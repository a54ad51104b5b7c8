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

// ---------------------------------------------------------------------------
// 4-bit cache: integer dot products.
//
// Scores: q is held as 15-bit fixed point q_i = round(q * 2^(14-e)) (e the
// exponent of max|q|), split into a signed high byte and an unsigned low byte
// (q_i = 256 hi + lo).  A 32-bit word of 8 codes (canonical nibbles) gives the
// even elements as bytes by one mask and the odd ones by a shift and a mask,
// so dp4a forms sum_e q_i,e code_e exactly in integers; per group
//   q . x_hat = scale * 2^(e-14) * sum_e q_i,e code_e + min * sum_e q_e.
// Values: with p_t = exp(s_t - max), each group's weights w_t = p_t * scale_t
// are held as 16-bit fixed point w_i = round(w_t * 65535 / max_t w_t), packed
// per block of 8 tokens into even/odd x high/low byte words in shared memory.
// The V codes are token-interleaved (nibble k of word (block, dim) = token
// 8*block + k), so dp4a weights 4 tokens of one dimension at a time:
//   sum_t p_t x_hat_t,e = max_w/65535 * sum_t w_i,t code_t,e + sum_t p_t min_t.
// Per element that is about one integer instruction instead of a conversion
// and a floating-point multiply-add.
// ---------------------------------------------------------------------------
constexpr int kStatN = 5;  // S, pm[2], wmax[2]
constexpr int kUnroll = 4;  // independent 16-byte loads in flight per lane in the K and V passes

__device__ __forceinline__ void block_reduce_stats(float (&v)[kStatN], float (*red)[kStatN]) {
#pragma unroll
  for (int k = 0; k < kStatN; ++k) {
    const bool is_max = k >= 3;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float other = __shfl_xor_sync(0xffffffffu, v[k], o);
      v[k] = is_max ? fmaxf(v[k], other) : v[k] + other;
    }
  }
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0)
#pragma unroll
    for (int k = 0; k < kStatN; ++k) red[w][k] = v[k];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kStatN; ++k) {
    float r = red[0][k];
    for (int i = 1; i < kThreads / 32; ++i) r = k >= 3 ? fmaxf(r, red[i][k]) : r + red[i][k];
    v[k] = r;
  }
}

template <int NW>
__device__ __forceinline__ void load_words(const uint32_t* p, uint32_t (&w)[NW]) {
  if constexpr (NW == 4) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    w[0] = u.x; w[1] = u.y;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) attn_decode_q4_kernel(const __half* __restrict__ q, int ldq, KvView kv,
                                                                  int heads, int len, __half* __restrict__ out,
                                                                  int ldo, float inv_sqrt_d) {
  constexpr int DPL = D / 4;   // score pass: dimensions per lane (one group)
  constexpr int NW = DPL / 8;  // code words per lane per token
  constexpr int G = D / 64;    // groups per head row
  constexpr int DPV = D / 32;  // value pass: dimensions per lane
  extern __shared__ float sc[];  // [len] scores, then probabilities
  uint4* wpk = reinterpret_cast<uint4*>(sc + ((len + 3) & ~3));  // [blocks][G] packed weights
  __shared__ float red[kThreads / 32][kStatN];
  __shared__ float partv[kThreads / 32][D];
  const int j = blockIdx.x, i = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = lane & 3;
  const int g = (c * DPL) / 64;
  const size_t hr = static_cast<size_t>(i) * heads + j;
  const uint32_t* kw = reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(kv.k) + hr * kv.max_len * (D / 2));
  const __half2* km = static_cast<const __half2*>(kv.k_meta) + hr * kv.max_len * G;
  const __half2* vm = static_cast<const __half2*>(kv.v_meta) + hr * kv.max_len * G;
  const uint32_t* vw = static_cast<const uint32_t*>(kv.v) + hr * (kv_pad_len(kv.max_len) / 8) * D;

  // q slice of this lane as fp32, its sum, and the fixed-point bytes
  float qf[DPL];
  const __half* qp = q + static_cast<size_t>(i) * ldq + j * D + c * DPL;
#pragma unroll
  for (int e = 0; e < DPL; e += 2) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(qp + e));
    qf[e] = f.x;
    qf[e + 1] = f.y;
  }
  float qsum = 0.f, qmax = 0.f;
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    qsum += qf[e];
    qmax = fmaxf(qmax, fabsf(qf[e]));
  }
  qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, 1));
  qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, 2));
  int qexp = 0;
  frexpf(qmax, &qexp);
  const float qscale = ldexpf(1.0f, 14 - qexp);
  const float inv_qscale = ldexpf(1.0f, qexp - 14);
  int qh_e[NW], qh_o[NW];
  uint32_t ql_e[NW], ql_o[NW];
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    qh_e[w] = qh_o[w] = 0;
    ql_e[w] = ql_o[w] = 0u;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const int ie = __float2int_rn(qf[8 * w + 2 * n] * qscale);
      const int io = __float2int_rn(qf[8 * w + 2 * n + 1] * qscale);
      qh_e[w] |= ((ie >> 8) & 0xFF) << (8 * n);
      qh_o[w] |= ((io >> 8) & 0xFF) << (8 * n);
      ql_e[w] |= static_cast<uint32_t>(ie & 0xFF) << (8 * n);
      ql_o[w] |= static_cast<uint32_t>(io & 0xFF) << (8 * n);
    }
  }

  // pass 1: scores, 8 tokens per warp, 4 lanes per token.  kUnroll groups of
  // tokens are loaded before any is used, so each warp keeps several 16-byte
  // loads per lane in flight (the pass is bound by load latency otherwise).
  float mx = -INFINITY;
  constexpr int kStride = kThreads / 4;  // tokens per block-wide step
  for (int base = warp * 8; base < len; base += kUnroll * kStride) {
    uint32_t cw[kUnroll][NW];
    __half2 msh[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = base + u * kStride + (lane >> 2);
      if (t < len) {
        load_words<NW>(kw + static_cast<size_t>(t) * (D / 8) + c * NW, cw[u]);
        msh[u] = km[static_cast<size_t>(t) * G + g];  // (min, scale)
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = base + u * kStride + (lane >> 2);
      const bool valid = t < len;
      float partial = 0.f;
      if (valid) {
        int dh = 0;
        uint32_t dl = 0u;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const uint32_t lo = cw[u][w] & 0x0F0F0F0Fu;
          const uint32_t hi = (cw[u][w] >> 4) & 0x0F0F0F0Fu;
          dh = __dp4a(static_cast<int>(lo), qh_e[w], dh);
          dh = __dp4a(static_cast<int>(hi), qh_o[w], dh);
          dl = __dp4a(lo, ql_e[w], dl);
          dl = __dp4a(hi, ql_o[w], dl);
        }
        const float dot = (static_cast<float>(dh) * 256.0f + static_cast<float>(dl)) * inv_qscale;
        const float2 ms = __half22float2(msh[u]);
        partial = ms.y * dot + ms.x * qsum;
      }
      partial += __shfl_xor_sync(0xffffffffu, partial, 1);
      partial += __shfl_xor_sync(0xffffffffu, partial, 2);
      if (valid) {
        const float s = partial * inv_sqrt_d;
        if (c == 0) sc[t] = s;
        mx = fmaxf(mx, s);
      }
    }
  }
  const float M = block_reduce(mx, &red[0][0], true);

  // pass 2a: probabilities, their sum, per-group sum p*min and max p*scale
  float st[kStatN] = {0.f, 0.f, 0.f, 0.f, 0.f};
  for (int t = threadIdx.x; t < len; t += kThreads) {
    const float p = __expf(sc[t] - M);
    sc[t] = p;
    st[0] += p;
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      const float2 ms = __half22float2(vm[static_cast<size_t>(t) * G + gg]);
      st[1 + gg] += p * ms.x;
      st[3 + gg] = fmaxf(st[3 + gg], p * ms.y);
    }
  }
  block_reduce_stats(st, red);
  const float S = st[0];

  // pass 2b: 16-bit fixed-point weights packed per (8-token block, group)
  const int nblk = (len + 7) / 8;
  for (int idx = threadIdx.x; idx < nblk * G; idx += kThreads) {
    const int blk = idx / G, gg = idx % G;
    const float wq = st[3 + gg] > 0.f ? 65535.0f / st[3 + gg] : 0.f;
    uint32_t le = 0u, lo = 0u, he = 0u, ho = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int t = blk * 8 + k;
      uint32_t wi = 0u;
      if (t < len) {
        const float sv = __high2float(vm[static_cast<size_t>(t) * G + gg]);  // scale
        wi = min(65535u, __float2uint_rn(sc[t] * sv * wq));
      }
      const int sh = 8 * (k >> 1);
      if (k & 1) {
        lo |= (wi & 0xFFu) << sh;
        ho |= (wi >> 8) << sh;
      } else {
        le |= (wi & 0xFFu) << sh;
        he |= (wi >> 8) << sh;
      }
    }
    wpk[idx] = make_uint4(le, lo, he, ho);
  }
  __syncthreads();

  // pass 3: values, one 8-token block per warp step, DPV dimensions per lane
  const int gv = (lane * DPV) / 64;
  uint32_t ah[DPV], al[DPV];
#pragma unroll
  for (int e = 0; e < DPV; ++e) ah[e] = al[e] = 0u;
  constexpr int kWarps = kThreads / 32;
  for (int blk0 = warp; blk0 < nblk; blk0 += kUnroll * kWarps) {
    uint32_t vwd[kUnroll][DPV];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int blk = blk0 + u * kWarps;
      if (blk < nblk) load_words<DPV>(vw + static_cast<size_t>(blk) * D + lane * DPV, vwd[u]);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int blk = blk0 + u * kWarps;
      if (blk >= nblk) break;
      const uint4 wp = wpk[blk * G + gv];
#pragma unroll
      for (int e = 0; e < DPV; ++e) {
        const uint32_t lo = vwd[u][e] & 0x0F0F0F0Fu;
        const uint32_t hi = (vwd[u][e] >> 4) & 0x0F0F0F0Fu;
        al[e] = __dp4a(lo, wp.x, al[e]);
        al[e] = __dp4a(hi, wp.y, al[e]);
        ah[e] = __dp4a(lo, wp.z, ah[e]);
        ah[e] = __dp4a(hi, wp.w, ah[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < DPV; ++e)
    partv[warp][lane * DPV + e] = static_cast<float>(ah[e]) * 256.0f + static_cast<float>(al[e]);
  __syncthreads();
  const float invS = 1.0f / S;
  for (int e = threadIdx.x; e < D; e += kThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) v += partv[w][e];
    const int gg = e / 64;
    const float o = v * (st[3 + gg] / 65535.0f) + st[1 + gg];
    out[static_cast<size_t>(i) * ldo + j * D + e] = __float2half_rn(o * invS);
  }
}

template <int D>
cudaError_t launch_q4(const __half* q, int ldq, const KvView& kv, int b, int heads, int len, __half* out, int ldo,
                      cudaStream_t s) {
  const size_t smem = static_cast<size_t>((len + 3) & ~3) * sizeof(float) +
                      static_cast<size_t>((len + 7) / 8) * (D / 64) * sizeof(uint4);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(attn_decode_q4_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(heads, b);
  attn_decode_q4_kernel<D><<<grid, kThreads, smem, s>>>(q, ldq, kv, heads, len, out, ldo,
                                                        1.0f / sqrtf(static_cast<float>(D)));
  return launched();
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
    return kv_bits == 4 ? launch_q4<128>(q, ldq, kv, b, heads, len, out, ldo, s)
                        : launch_one<128, 16>(q, ldq, kv, b, heads, len, out, ldo, s);
  return kv_bits == 4 ? launch_q4<64>(q, ldq, kv, b, heads, len, out, ldo, s)
                      : launch_one<64, 16>(q, ldq, kv, b, heads, len, out, ldo, s);
}

}  // namespace flexq

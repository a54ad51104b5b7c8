// Row-wise kernels: LayerNorm, word + positional embedding, greedy argmax.
//
// LayerNorm: one per block of the pre-LN OPT layer and a final one before the
// tied LM head ("FlexGen: High-Throughput Generative Inference ..." walk-through,
// section "内存占用分析": gamma, beta in R^h per LayerNorm; survey notes,
// "Transformer-Styles LLMs").  fp32 statistics, biased variance, two passes
// over registers (mean, then sum of squared deviations), fp16 out.
// Embedding: x0 = E[token] + P[position] (survey notes: word embedding plus
// positional embedding before the first block); the decode variant also
// applies the first layer's LN1 to the row it holds.
// Argmax: greedy choice over the vocabulary, lowest index among equal maxima.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace flexq {
namespace {

constexpr int kLnThreads = 128;
constexpr int kLnMaxVec = 12;  // h <= 128 threads * 12 vectors * 8 = 12288

__device__ __forceinline__ float block_sum_128(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if (lane_id() == 0) red[w] = v;
  __syncthreads();
  return red[0] + red[1] + red[2] + red[3];
}

__global__ void __launch_bounds__(kLnThreads) layernorm_kernel(const __half* __restrict__ x, int ldx,
                                                               const __half* __restrict__ g,
                                                               const __half* __restrict__ bta,
                                                               __half* __restrict__ y, int ldy, int h,
                                                               float eps) {
  __shared__ float red[4];
  const int nvec = h / 8;
  const __half* xr = x + static_cast<size_t>(blockIdx.x) * ldx;
  float v[kLnMaxVec][8];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < kLnMaxVec; ++i) {
    const int vi = threadIdx.x + i * kLnThreads;
    if (vi < nvec) {
      const uint4 u = reinterpret_cast<const uint4*>(xr)[vi];
      const __half2* h2 = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h2[e]);
        v[i][2 * e] = f.x;
        v[i][2 * e + 1] = f.y;
        sum += f.x + f.y;
      }
    }
  }
  const float mean = block_sum_128(sum, red) / static_cast<float>(h);
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < kLnMaxVec; ++i) {
    const int vi = threadIdx.x + i * kLnThreads;
    if (vi < nvec) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float dlt = v[i][e] - mean;
        sq += dlt * dlt;
      }
    }
  }
  const float var = block_sum_128(sq, red) / static_cast<float>(h);
  const float rstd = 1.0f / sqrtf(var + eps);
  __half* yr = y + static_cast<size_t>(blockIdx.x) * ldy;
#pragma unroll
  for (int i = 0; i < kLnMaxVec; ++i) {
    const int vi = threadIdx.x + i * kLnThreads;
    if (vi < nvec) {
      const uint4 gu = reinterpret_cast<const uint4*>(g)[vi];
      const uint4 bu = reinterpret_cast<const uint4*>(bta)[vi];
      const __half2* g2 = reinterpret_cast<const __half2*>(&gu);
      const __half2* b2 = reinterpret_cast<const __half2*>(&bu);
      __align__(16) __half2 o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 gf = __half22float2(g2[e]);
        const float2 bf = __half22float2(b2[e]);
        o[e] = __floats2half2_rn((v[i][2 * e] - mean) * rstd * gf.x + bf.x,
                                 (v[i][2 * e + 1] - mean) * rstd * gf.y + bf.y);
      }
      reinterpret_cast<uint4*>(yr)[vi] = *reinterpret_cast<const uint4*>(o);
    }
  }
}

// Eight consecutive elements (8 vi .. 8 vi + 7) of row `id` of the word
// embedding E [vocab][h]: fp16, or the 4-bit tiled layout of the linear
// layers (row id in tile id / 128, 64-wide k-block 8 vi / 64; nibble order
// within a 32-bit word: element e in nibble (e >> 1) + 4 (e & 1)), whose
// values are x_hat = fp16_rn(fp32(code * scale) + min), the codec's
// dequantizer ("FlexGen研究学术报告" section 三(C): dequantized to FP16).
__device__ __forceinline__ uint4 embed_row8(const void* E, int embed_bits, int id, int vi, int h) {
  if (embed_bits == 16) return reinterpret_cast<const uint4*>(static_cast<const __half*>(E) + static_cast<size_t>(id) * h)[vi];
  const int e0 = vi * 8, kb = e0 / 64;
  const uint8_t* tile = static_cast<const uint8_t*>(E) +
                        (static_cast<size_t>(id / kTileRows) * (h / kGroup) + kb) * kTileBytes;
  const int row = id % kTileRows;
  const uint32_t w = *reinterpret_cast<const uint32_t*>(tile + row * 32 + ((e0 % 64) / 8) * 4);
  const float2 ms = __half22float2(*reinterpret_cast<const __half2*>(tile + kTileCodeBytes + row * 4));
  uint32_t out[4];
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    const float q0 = static_cast<float>((w >> (4 * ((e >> 1) + 0))) & 0xFu);
    const float q1 = static_cast<float>((w >> (4 * ((e >> 1) + 4))) & 0xFu);
    const __half2 v = __halves2half2(__float2half_rn(__fadd_rn(__fmul_rn(q0, ms.y), ms.x)),
                                     __float2half_rn(__fadd_rn(__fmul_rn(q1, ms.y), ms.x)));
    out[e / 2] = *reinterpret_cast<const uint32_t*>(&v);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

__global__ void embed_kernel(const int32_t* __restrict__ tok, int ld_tok, int ntok,
                             const void* __restrict__ E, int embed_bits, int vocab, const __half* __restrict__ P,
                             int pos0, int h, __half* __restrict__ x, uint32_t* err) {
  const int r = blockIdx.x;  // i * ntok + t
  const int i = r / ntok, t = r % ntok;
  int id = tok[static_cast<size_t>(i) * ld_tok + t];
  if (id < 0 || id >= vocab) {  // a bad token id is reported, never dereferenced
    if (threadIdx.x == 0) set_error(err, DEV_BAD_ARGUMENT);
    id = 0;
  }
  const uint4* pr = reinterpret_cast<const uint4*>(P + static_cast<size_t>(pos0 + t) * h);
  uint4* xr = reinterpret_cast<uint4*>(x + static_cast<size_t>(r) * h);
  for (int v = threadIdx.x; v < h / 8; v += blockDim.x) {
    const uint4 a = embed_row8(E, embed_bits, id, v, h), b = pr[v];
    const __half2* a2 = reinterpret_cast<const __half2*>(&a);
    const __half2* b2 = reinterpret_cast<const __half2*>(&b);
    __align__(16) __half2 o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa = __half22float2(a2[e]);
      const float2 fb = __half22float2(b2[e]);
      o[e] = __floats2half2_rn(fa.x + fb.x, fa.y + fb.y);
    }
    xr[v] = *reinterpret_cast<const uint4*>(o);
  }
}

// Decode embedding fused with the first layer's LN1: one CTA per sequence;
// x = fp16(E[tok] + P[pos]) is stored and, from those fp16 values held in
// registers, u = LN(x) with the statistics of layernorm_kernel.
__global__ void __launch_bounds__(kLnThreads) embed_ln_kernel(const int32_t* __restrict__ tok, int ld_tok,
                                                              const void* __restrict__ E, int embed_bits, int vocab,
                                                              const __half* __restrict__ P, int pos, int h,
                                                              __half* __restrict__ x, const __half* __restrict__ g,
                                                              const __half* __restrict__ bta, float eps,
                                                              __half* __restrict__ u, uint32_t* err) {
  __shared__ float red[4];
  const int r = blockIdx.x;
  int id = tok[static_cast<size_t>(r) * ld_tok];
  if (id < 0 || id >= vocab) {  // a bad token id is reported, never dereferenced
    if (threadIdx.x == 0) set_error(err, DEV_BAD_ARGUMENT);
    id = 0;
  }
  const uint4* pr = reinterpret_cast<const uint4*>(P + static_cast<size_t>(pos) * h);
  uint4* xr = reinterpret_cast<uint4*>(x + static_cast<size_t>(r) * h);
  const int nvec = h / 8;
  float v[kLnMaxVec][8];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < kLnMaxVec; ++i) {
    const int vi = threadIdx.x + i * kLnThreads;
    if (vi < nvec) {
      const uint4 a = embed_row8(E, embed_bits, id, vi, h), b = pr[vi];
      const __half2* a2 = reinterpret_cast<const __half2*>(&a);
      const __half2* b2 = reinterpret_cast<const __half2*>(&b);
      __align__(16) __half2 o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __half22float2(a2[e]);
        const float2 fb = __half22float2(b2[e]);
        o[e] = __floats2half2_rn(fa.x + fb.x, fa.y + fb.y);
        const float2 f = __half22float2(o[e]);
        v[i][2 * e] = f.x;
        v[i][2 * e + 1] = f.y;
        sum += f.x + f.y;
      }
      xr[vi] = *reinterpret_cast<const uint4*>(o);
    }
  }
  const float mean = block_sum_128(sum, red) / static_cast<float>(h);
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < kLnMaxVec; ++i) {
    if (threadIdx.x + i * kLnThreads < nvec) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float dlt = v[i][e] - mean;
        sq += dlt * dlt;
      }
    }
  }
  const float var = block_sum_128(sq, red) / static_cast<float>(h);
  const float rstd = 1.0f / sqrtf(var + eps);
  __half* ur = u + static_cast<size_t>(r) * h;
#pragma unroll
  for (int i = 0; i < kLnMaxVec; ++i) {
    const int vi = threadIdx.x + i * kLnThreads;
    if (vi < nvec) {
      const uint4 gu = reinterpret_cast<const uint4*>(g)[vi];
      const uint4 bu = reinterpret_cast<const uint4*>(bta)[vi];
      const __half2* g2 = reinterpret_cast<const __half2*>(&gu);
      const __half2* b2 = reinterpret_cast<const __half2*>(&bu);
      __align__(16) __half2 o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 gf = __half22float2(g2[e]);
        const float2 bf = __half22float2(b2[e]);
        o[e] = __floats2half2_rn((v[i][2 * e] - mean) * rstd * gf.x + bf.x,
                                 (v[i][2 * e + 1] - mean) * rstd * gf.y + bf.y);
      }
      reinterpret_cast<uint4*>(ur)[vi] = *reinterpret_cast<const uint4*>(o);
    }
  }
}

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

__global__ void argmax_kernel(const float* __restrict__ logits, int vocab, int ld,
                              int32_t* __restrict__ out, int ld_out) {
  __shared__ float sv[32];
  __shared__ int si[32];
  const float* row = logits + static_cast<size_t>(blockIdx.x) * ld;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int i = threadIdx.x; i < vocab; i += blockDim.x) {
    const float v = row[i];
    if (better(v, i, bv, bi)) { bv = v; bi = i; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
  }
  const int w = threadIdx.x >> 5;
  if (lane_id() == 0) { sv[w] = bv; si[w] = bi; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < static_cast<int>(blockDim.x >> 5); ++k)
      if (better(sv[k], si[k], bv, bi)) { bv = sv[k]; bi = si[k]; }
    out[static_cast<size_t>(blockIdx.x) * ld_out] = bi == 0x7fffffff ? 0 : bi;
  }
}

}  // namespace

cudaError_t launch_layernorm(const __half* x, int ldx, const __half* g, const __half* bta, __half* y,
                             int ldy, int rows, int h, float eps, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  layernorm_kernel<<<rows, kLnThreads, 0, s>>>(x, ldx, g, bta, y, ldy, h, eps);
  return launched();
}

cudaError_t launch_embed(const int32_t* tok, int ld_tok, int b, int ntok, const void* E, int embed_bits,
                         int vocab, const __half* P, int pos0, int h, __half* x, cudaStream_t s) {
  if (b == 0 || ntok == 0) return cudaSuccess;
  embed_kernel<<<b * ntok, 128, 0, s>>>(tok, ld_tok, ntok, E, embed_bits, vocab, P, pos0, h, x, runtime().err);
  return launched();
}

cudaError_t launch_embed_ln(const int32_t* tok, int ld_tok, int b, const void* E, int embed_bits, int vocab,
                            const __half* P, int pos, int h, __half* x, const __half* g,
                            const __half* bta, float eps, __half* u, cudaStream_t s) {
  if (b == 0) return cudaSuccess;
  embed_ln_kernel<<<b, kLnThreads, 0, s>>>(tok, ld_tok, E, embed_bits, vocab, P, pos, h, x, g, bta, eps, u,
                                           runtime().err);
  return launched();
}

cudaError_t launch_argmax(const float* logits, int rows, int vocab, int ld, int32_t* out,
                          int ld_out, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  argmax_kernel<<<rows, 512, 0, s>>>(logits, vocab, ld, out, ld_out);
  return launched();
}

}  // namespace flexq

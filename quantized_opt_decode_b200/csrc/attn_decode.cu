// Decode attention over the KV cache: for each (sequence, head),
//   o = softmax(q K^T / sqrt(d)) V  over the cached slots 0..len-1,
// the decode equation t_out = softmax(t_Q x_K^T / sqrt(.)) x_V W_O + t of the
// FlexGen walk-through (section "P/D阶段计算") in the per-head form of the
// survey notes' eq. (2), with K and V stored in the group-wise 4-bit format of
// "FlexGen研究学术报告" section 三(C) (or fp16).
//
// Two pipelined kernels, one per cache format, that stream each head's rows
// through shared memory (below).  4-bit codes are dequantized without
// materialising x_hat:
//   q . x_hat = scale * sum_e q_e code_e + min * sum_e q_e   (per group)
//   sum_t p_t x_hat_t = sum_t (p_t scale_t) code_t + sum_t p_t min_t,
// which is the dequantized value code * scale + min before its fp16 rounding.
// K and V are each read once.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "quant_common.cuh"

namespace flexq {
namespace {

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

// ---------------------------------------------------------------------------
// 4-bit cache, one CTA per (head, sequence) (the decode step's shape: many
// sequences): integer dot products over the cache read straight from HBM.
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
// Pass 1 (scores, six 16-byte loads in flight per lane), pass 2 (softmax
// weights and their fixed-point packing), pass 3 (values, likewise six loads
// in flight).  In a decode step the warps first append the token's K/V rows
// to the cache (quantize on append, one warp per 64-element group), so the
// step needs no separate launch.
// ---------------------------------------------------------------------------
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

constexpr int kStatN = 5;  // S, pm[2], wmax[2]
// Independent 16-byte loads in flight per lane in the K and V passes; with 7
// CTAs per SM (72 registers) six was measured faster than four at 8 CTAs and
// than eight at 6 CTAs (OPT-30B and OPT-175B decode shapes, KV length 528
// and 1040).
constexpr int kUnroll = 6;
constexpr int kMinBlocks = 7;

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

template <int D>
__global__ void __launch_bounds__(kThreads, kMinBlocks) attn_decode_q4_kernel(const __half* __restrict__ q, int ldq, KvView kv,
                                                                  int heads, int len, __half* __restrict__ out,
                                                                  int ldo, float inv_sqrt_d, AppendRow app) {
  pdl_wait();  // q, the cache and the outputs follow the stream's earlier kernels
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

  // decode: this token's K/V rows enter the cache before the passes read it
  if (app.pos >= 0) {
    append_group_q4<D>(app, kv, i, j, heads, warp, lane);
    __syncthreads();
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


// ---------------------------------------------------------------------------
// 4-bit cache, split along the cache (few sequences, long caches): streamed
// through shared memory, integer dot products.
//
// One CTA per (head, sequence, split): a producer warp streams the head's
// rows 128 tokens at a time through a ring of shared-memory stages with
// cp.async.bulk (K codes, K (min, scale), V words, V (min, scale) are each
// contiguous per head, so a chunk is four bulk copies); four compute warps
// take 32 tokens (four V blocks) of every chunk each and keep their own
// online-softmax state (running max m, sum l, and the weighted sum of V), so
// a chunk needs no block-wide barrier; the warps (and, for long caches split
// across CTAs, the splits) are merged at the end in a fixed order.
//
// Scores: q is held as 15-bit fixed point q_i = round(q * 2^(14-e)) (e the
// exponent of max|q| over the head row), split into a signed high byte and an unsigned low byte
// (q_i = 256 hi + lo).  A 32-bit word of 8 codes (canonical nibbles) gives the
// even elements as bytes by one mask and the odd ones by a shift and a mask,
// so dp4a forms sum_e q_i,e code_e exactly in integers; per group
//   q . x_hat = scale * 2^(e-14) * sum_e q_i,e code_e + min * sum_e q_e.
// Values: with p_t = exp(s_t - m), the weights w_t = p_t * scale_t of each
// group are held, per warp and chunk, as 16-bit fixed point
// w_i = round(w_t * 65535 / max w_t), packed per block of 8 tokens into
// even/odd x high/low byte words.  The V codes are token-interleaved (nibble
// k of word (block, dim) = token 8*block + k), so dp4a weights 4 tokens of one
// dimension at a time:
//   sum_t p_t x_hat_t,e = max w/65535 * sum_t w_i,t code_t,e + sum_t p_t min_t.
// ---------------------------------------------------------------------------
constexpr int kChunk = 128;      // tokens per pipeline stage (16 V blocks)
constexpr int kComputeWarps = 4; // 32 tokens (4 V blocks) of each chunk per warp
constexpr int kQ4Threads = 32 * (kComputeWarps + 1);
constexpr int kMaxSplits = 16;

// Shared-memory stage of one chunk.  The (min, scale) regions keep 16 bytes
// of slack: a head's metadata row starts wherever hr * max_len * 4G bytes
// puts it, so it lands in shared memory at the same offset modulo 16, which
// lets the bulk copy move its 16-byte-aligned middle.
template <int D>
struct Q4Stage {
  static constexpr int G = D / 64;
  static constexpr int kc = kChunk * D / 2;           // K codes
  static constexpr int km = kChunk * G * 4 + 16;      // K (min, scale)
  static constexpr int vw = kChunk / 8 * D * 4;       // V words
  static constexpr int vm = kChunk * G * 4 + 16;      // V (min, scale)
  static constexpr int bytes = kc + km + vw + vm;
  static constexpr int stages = D == 128 ? 3 : 4;
};

// Copies `bytes` (a multiple of 4) from src to dst, where dst and src agree
// modulo 16: the 16-byte-aligned middle by one bulk copy counted on `bar`
// (issued by the caller with the returned (offset, size)), the unaligned
// head and tail by plain loads and stores of the calling thread, done here
// so that the caller's mbarrier arrival publishes them.
__device__ __forceinline__ uint2 copy_edges(uint8_t* dst, const uint8_t* src, uint32_t bytes) {
  const uint32_t mis = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(src) & 15u);
  uint32_t lead = (16u - mis) & 15u;
  if (lead > bytes) lead = bytes;
  const uint32_t main = (bytes - lead) & ~15u;
  for (uint32_t o = 0; o < lead; o += 4)
    *reinterpret_cast<uint32_t*>(dst + o) = *reinterpret_cast<const uint32_t*>(src + o);
  for (uint32_t o = lead + main; o < bytes; o += 4)
    *reinterpret_cast<uint32_t*>(dst + o) = *reinterpret_cast<const uint32_t*>(src + o);
  return make_uint2(lead, main);
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  if (bytes == 0) return;
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Merges the compute warps' online-softmax states (running max, sum, and
// weighted value sums) in warp order; with several splits along the cache
// the merged state goes to `part` and the last split to arrive merges all of
// them in split order (results independent of timing) and resets the
// (sequence, head) counter.  Every thread of the CTA calls it after the
// warps have published cm / cl / cacc.
template <int D>
__device__ void merge_and_store(const float* cm, const float* cl, const float (*cacc)[D], __half* __restrict__ out,
                                int ldo, int i, int j, size_t hr, int z, float* __restrict__ part,
                                int* __restrict__ ctr, int* last_flag) {
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kComputeWarps; ++w) M = fmaxf(M, cm[w]);
  float ws[kComputeWarps];
  float Lsum = 0.f;
#pragma unroll
  for (int w = 0; w < kComputeWarps; ++w) {
    ws[w] = cm[w] == -INFINITY ? 0.f : __expf(cm[w] - M);
    Lsum += cl[w] * ws[w];
  }
  const int S = gridDim.z;
  if (S == 1) {
    for (int e = threadIdx.x; e < D; e += blockDim.x) {
      float o = 0.f;
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) o += cacc[w][e] * ws[w];
      out[static_cast<size_t>(i) * ldo + j * D + e] = __float2half_rn(o / Lsum);
    }
    return;
  }
  float* mine = part + (hr * S + z) * (D + 2);
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kComputeWarps; ++w) o += cacc[w][e] * ws[w];
    __stcg(mine + 2 + e, o);
  }
  if (threadIdx.x == 0) {
    __stcg(mine, M);
    __stcg(mine + 1, Lsum);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int old = atomicAdd(ctr + hr, 1);
    *last_flag = old == S - 1;
    if (*last_flag) ctr[hr] = 0;  // every split has counted in: leave the counter zero
    __threadfence();
  }
  __syncthreads();
  if (!*last_flag) return;
  const float* all = part + hr * S * (D + 2);
  float Mz = -INFINITY;
  for (int zz = 0; zz < S; ++zz) Mz = fmaxf(Mz, __ldcg(all + zz * (D + 2)));
  float Lz = 0.f;
  for (int zz = 0; zz < S; ++zz) {
    const float mz = __ldcg(all + zz * (D + 2));
    if (mz != -INFINITY) Lz += __ldcg(all + zz * (D + 2) + 1) * __expf(mz - Mz);
  }
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float o = 0.f;
    for (int zz = 0; zz < S; ++zz) {
      const float mz = __ldcg(all + zz * (D + 2));
      if (mz != -INFINITY) o += __ldcg(all + zz * (D + 2) + 2 + e) * __expf(mz - Mz);
    }
    out[static_cast<size_t>(i) * ldo + j * D + e] = __float2half_rn(o / Lz);
  }
}

template <int D>
__global__ void __launch_bounds__(kQ4Threads) attn_decode_q4_split_kernel(const __half* __restrict__ q, int ldq, KvView kv,
                                                                    int heads, int len, __half* __restrict__ out,
                                                                    int ldo, float inv_sqrt_d, int span,
                                                                    float* __restrict__ part, int* __restrict__ ctr,
                                                                    uint64_t wait_ns, uint32_t* err) {
  pdl_wait();  // q, the cache and the outputs follow the stream's earlier kernels
  using L = Q4Stage<D>;
  constexpr int G = L::G;
  constexpr int NS = L::stages;
  constexpr int DPL = D / 4;   // score pass: dimensions per lane (inside one group)
  constexpr int NW = DPL / 8;  // code words per lane and token
  constexpr int DPV = D / 32;  // value pass: dimensions per lane
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[NS], empty[NS];
  __shared__ float cm[kComputeWarps], cl[kComputeWarps];
  __shared__ float cacc[kComputeWarps][D];
  __shared__ int last_flag;
  const int j = blockIdx.x, i = blockIdx.y, z = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t hr = static_cast<size_t>(i) * heads + j;
  const int t_begin = z * span;
  const int t_end = min(len, t_begin + span);
  const int n_chunks = t_end > t_begin ? (t_end - t_begin + kChunk - 1) / kChunk : 0;

  if (threadIdx.x == 0) {
    for (int st = 0; st < NS; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kComputeWarps);
    }
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == kComputeWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint8_t* kc = static_cast<const uint8_t*>(kv.k) + hr * kv.max_len * (D / 2);
      const uint8_t* km = static_cast<const uint8_t*>(kv.k_meta) + hr * kv.max_len * G * 4;
      const uint8_t* vw = static_cast<const uint8_t*>(kv.v) + hr * (kv_pad_len(kv.max_len) / 8) * D * 4;
      const uint8_t* vm = static_cast<const uint8_t*>(kv.v_meta) + hr * kv.max_len * G * 4;
      const uint32_t km_off = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(km) & 15u);
      const uint32_t vm_off = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(vm) & 15u);
      bool stop = false;
      for (int c = 0; c < n_chunks && !stop; ++c) {
        const int st = c % NS;
        const uint32_t ph = static_cast<uint32_t>(c / NS) & 1u;
        if (!mbar_wait(&empty[st], ph ^ 1u, wait_ns)) {
          set_error(err, DEV_TIMEOUT_PRODUCER);
          stop = true;
          break;
        }
        const int t0 = t_begin + c * kChunk;
        const int nt = min(kChunk, t_end - t0);
        uint8_t* sb = ring + st * L::bytes;
        // K codes and V words are 16-byte aligned per head row and token
        // (d/2 and 4d bytes); the metadata rows keep their offset modulo 16
        const uint32_t b_kc = static_cast<uint32_t>(nt) * (D / 2);
        const uint32_t b_vw = static_cast<uint32_t>((nt + 7) / 8) * D * 4;
        const uint8_t* km_src = km + static_cast<size_t>(t0) * G * 4;
        const uint8_t* vm_src = vm + static_cast<size_t>(t0) * G * 4;
        uint8_t* km_dst = sb + L::kc + km_off;
        uint8_t* vm_dst = sb + L::kc + L::km + L::vw + vm_off;
        const uint2 ek = copy_edges(km_dst, km_src, nt * G * 4);
        const uint2 ev = copy_edges(vm_dst, vm_src, nt * G * 4);
        mbar_arrive_expect_tx(&full[st], b_kc + ek.y + b_vw + ev.y);
        bulk_g2s(sb, kc + static_cast<size_t>(t0) * (D / 2), b_kc, &full[st]);
        bulk_g2s(km_dst + ek.x, km_src + ek.x, ek.y, &full[st]);
        bulk_g2s(sb + L::kc + L::km, vw + static_cast<size_t>(t0 / 8) * D * 4, b_vw, &full[st]);
        bulk_g2s(vm_dst + ev.x, vm_src + ev.x, ev.y, &full[st]);
      }
      // never leave the CTA with bulk copies still landing in shared memory
      const uint64_t drain = wait_ns > 1000000000ull ? wait_ns : 1000000000ull;
      for (int c = max(0, n_chunks - NS); c < n_chunks; ++c)
        mbar_wait(&full[c % NS], static_cast<uint32_t>(c / NS) & 1u, drain);
    }
  } else {
    // ------------------------------------------------------------ compute
    const int tk = lane >> 2, cq = lane & 3;
    const int g = (cq * DPL) / 64;  // group of this lane's score dimensions
    const int gv = (lane * DPV) / 64;  // group of this lane's value dimensions
    // q slice of this lane as fp32, its sum, and the fixed-point bytes
    float qf[DPL];
    const __half* qp = q + static_cast<size_t>(i) * ldq + j * D + cq * DPL;
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

    // the metadata rows sit in shared memory at their global offset modulo 16
    const uint32_t km_off = static_cast<uint32_t>(
        reinterpret_cast<uintptr_t>(static_cast<const uint8_t*>(kv.k_meta) + hr * kv.max_len * G * 4) & 15u);
    const uint32_t vm_off = static_cast<uint32_t>(
        reinterpret_cast<uintptr_t>(static_cast<const uint8_t*>(kv.v_meta) + hr * kv.max_len * G * 4) & 15u);
    float m_run = -INFINITY, l_run = 0.f;
    float acc[DPV];
#pragma unroll
    for (int e = 0; e < DPV; ++e) acc[e] = 0.f;
    bool bad = false;
    for (int c = 0; c < n_chunks; ++c) {
      const int st = c % NS;
      if (!bad && !mbar_wait(&full[st], static_cast<uint32_t>(c / NS) & 1u, wait_ns)) {
        set_error(err, DEV_TIMEOUT_CONSUMER);
        bad = true;
      }
      const int nt = min(kChunk, t_end - (t_begin + c * kChunk));
      const uint8_t* sb = ring + st * L::bytes;
      const uint32_t* skc = reinterpret_cast<const uint32_t*>(sb);
      const __half2* skm = reinterpret_cast<const __half2*>(sb + L::kc + km_off);
      const uint32_t* svw = reinterpret_cast<const uint32_t*>(sb + L::kc + L::km);
      const __half2* svm = reinterpret_cast<const __half2*>(sb + L::kc + L::km + L::vw + vm_off);
      const int wt0 = warp * 32;
      float sc[4];
      float mloc = -INFINITY;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int tt = wt0 + u * 8 + tk;  // token inside the chunk
        float partial = 0.f;
        const bool valid = !bad && tt < nt;
        if (valid) {
          uint32_t cw[NW];
          load_words<NW>(skc + tt * (D / 8) + cq * NW, cw);
          int dh = 0;
          uint32_t dl = 0u;
#pragma unroll
          for (int w = 0; w < NW; ++w) {
            const uint32_t lo = cw[w] & 0x0F0F0F0Fu;
            const uint32_t hi = (cw[w] >> 4) & 0x0F0F0F0Fu;
            dh = __dp4a(static_cast<int>(lo), qh_e[w], dh);
            dh = __dp4a(static_cast<int>(hi), qh_o[w], dh);
            dl = __dp4a(lo, ql_e[w], dl);
            dl = __dp4a(hi, ql_o[w], dl);
          }
          const float dot = (static_cast<float>(dh) * 256.0f + static_cast<float>(dl)) * inv_qscale;
          const float2 ms = __half22float2(skm[tt * G + g]);  // (min, scale)
          partial = ms.y * dot + ms.x * qsum;
        }
        partial += __shfl_xor_sync(0xffffffffu, partial, 1);
        partial += __shfl_xor_sync(0xffffffffu, partial, 2);
        sc[u] = valid ? partial * inv_sqrt_d : -INFINITY;
        mloc = fmaxf(mloc, sc[u]);
      }
      const float m_c = warp_max(mloc);
      if (m_c != -INFINITY) {
        const float m_new = fmaxf(m_run, m_c);
        const float alpha = m_run == -INFINITY ? 0.f : __expf(m_run - m_new);
        // probabilities, their sum, and per group sum p*min and max p*scale
        float pr[4], vsc[4];
        float my_s = 0.f, my_pm = 0.f, my_wm = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int tt = wt0 + u * 8 + tk;
          pr[u] = sc[u] == -INFINITY ? 0.f : __expf(sc[u] - m_new);
          vsc[u] = 0.f;
          if (cq == 0) my_s += pr[u];
          if (cq < G && pr[u] > 0.f) {
            const float2 ms = __half22float2(svm[tt * G + cq]);
            my_pm += pr[u] * ms.x;
            vsc[u] = pr[u] * ms.y;
            my_wm = fmaxf(my_wm, vsc[u]);
          }
        }
        const float s_c = warp_sum(my_s);
        float pm[G], wm[G];
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          pm[gg] = warp_sum(cq == gg ? my_pm : 0.f);
          wm[gg] = warp_max(cq == gg ? my_wm : 0.f);
        }
        // 16-bit fixed-point weights of this lane's (token, group), then the
        // value pass over the warp's 4 blocks
        uint32_t al[DPV], ah[DPV];
#pragma unroll
        for (int e = 0; e < DPV; ++e) al[e] = ah[e] = 0u;
        const float wm_mine = cq == 0 ? wm[0] : wm[G - 1];  // this lane's group (cq < G)
        const float wq = cq < G && wm_mine > 0.f ? 65535.0f / wm_mine : 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t wi = cq < G ? min(65535u, __float2uint_rn(vsc[u] * wq)) : 0u;
          uint32_t le = 0u, lo = 0u, he = 0u, ho = 0u;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t w = __shfl_sync(0xffffffffu, wi, 4 * k + gv);
            const int sh = 8 * (k >> 1);
            if (k & 1) {
              lo |= (w & 0xFFu) << sh;
              ho |= (w >> 8) << sh;
            } else {
              le |= (w & 0xFFu) << sh;
              he |= (w >> 8) << sh;
            }
          }
          uint32_t vwd[DPV];
          load_words<DPV>(svw + (warp * 4 + u) * D + lane * DPV, vwd);
#pragma unroll
          for (int e = 0; e < DPV; ++e) {
            const uint32_t lo4 = vwd[e] & 0x0F0F0F0Fu;
            const uint32_t hi4 = (vwd[e] >> 4) & 0x0F0F0F0Fu;
            al[e] = __dp4a(lo4, le, al[e]);
            al[e] = __dp4a(hi4, lo, al[e]);
            ah[e] = __dp4a(lo4, he, ah[e]);
            ah[e] = __dp4a(hi4, ho, ah[e]);
          }
        }
        const float vscale = (gv == 0 ? wm[0] : wm[G - 1]) / 65535.0f;
        const float vmin = gv == 0 ? pm[0] : pm[G - 1];
#pragma unroll
        for (int e = 0; e < DPV; ++e)
          acc[e] = acc[e] * alpha + ((static_cast<float>(ah[e]) * 256.0f + static_cast<float>(al[e])) * vscale + vmin);
        l_run = l_run * alpha + s_c;
        m_run = m_new;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    if (lane == 0) {
      cm[warp] = m_run;
      cl[warp] = l_run;
    }
#pragma unroll
    for (int e = 0; e < DPV; ++e) cacc[warp][lane * DPV + e] = acc[e];
  }
  __syncthreads();

  merge_and_store<D>(cm, cl, cacc, out, ldo, i, j, hr, z, part, ctr, &last_flag);
}

template <int D>
cudaError_t launch_q4_dense(const __half* q, int ldq, const KvView& kv, int b, int heads, int len, __half* out,
                            int ldo, const AppendRow& app, cudaStream_t s) {
  const size_t smem = static_cast<size_t>((len + 3) & ~3) * sizeof(float) +
                      static_cast<size_t>((len + 7) / 8) * (D / 64) * sizeof(uint4);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(attn_decode_q4_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(heads, b);
  return launch_pdl(attn_decode_q4_kernel<D>, grid, dim3(kThreads), smem, s, q, ldq, kv, heads, len, out, ldo,
                    1.0f / sqrtf(static_cast<float>(D)), app);
}

template <int D>
cudaError_t launch_q4_split(const __half* q, int ldq, const KvView& kv, int b, int heads, int len, __half* out, int ldo,
                      int splits, float* part, int* ctr, cudaStream_t s) {
  using L = Q4Stage<D>;
  static cudaError_t attr = cudaFuncSetAttribute(attn_decode_q4_split_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 L::stages * L::bytes);
  if (attr != cudaSuccess) return attr;
  int span = (len + splits - 1) / splits;
  span = (span + kChunk - 1) / kChunk * kChunk;
  const int S = (len + span - 1) / span;
  dim3 grid(heads, b, S);
  return launch_pdl(attn_decode_q4_split_kernel<D>, grid, dim3(kQ4Threads), L::stages * L::bytes, s, q, ldq, kv,
                    heads, len, out, ldo, 1.0f / sqrtf(static_cast<float>(D)), span, part, ctr,
                    runtime().wait_limit_ns, runtime().err);
}

// ---------------------------------------------------------------------------
// fp16 cache: the same pipeline with fp16 K and V rows (T tokens per stage,
// K rows then V rows, two bulk copies), fp32 dot products and an fp32
// weighted sum of V per warp.
// ---------------------------------------------------------------------------
template <int D>
struct F16Stage {
  static constexpr int T = D == 128 ? 64 : 128;  // tokens per chunk
  static constexpr int row = D * 2;              // bytes per K or V row
  static constexpr int bytes = 2 * T * row;
  static constexpr int stages = 3;
};

template <int D>
__global__ void __launch_bounds__(kQ4Threads) attn_decode_f16_kernel(const __half* __restrict__ q, int ldq, KvView kv,
                                                                     int heads, int len, __half* __restrict__ out,
                                                                     int ldo, float inv_sqrt_d, int span,
                                                                     float* __restrict__ part, int* __restrict__ ctr,
                                                                     uint64_t wait_ns, uint32_t* err) {
  pdl_wait();  // q, the cache and the outputs follow the stream's earlier kernels
  using L = F16Stage<D>;
  constexpr int T = L::T, NS = L::stages;
  constexpr int TW = T / kComputeWarps;  // tokens per warp and chunk
  constexpr int DPL = D / 4;             // score pass: dimensions per lane
  constexpr int DPV = D / 32;            // value pass: dimensions per lane
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[NS], empty[NS];
  __shared__ float cm[kComputeWarps], cl[kComputeWarps];
  __shared__ float cacc[kComputeWarps][D];
  __shared__ int last_flag;
  const int j = blockIdx.x, i = blockIdx.y, z = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t hr = static_cast<size_t>(i) * heads + j;
  const int t_begin = z * span;
  const int t_end = min(len, t_begin + span);
  const int n_chunks = t_end > t_begin ? (t_end - t_begin + T - 1) / T : 0;

  if (threadIdx.x == 0) {
    for (int st = 0; st < NS; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kComputeWarps);
    }
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == kComputeWarps) {
    if (lane == 0) {
      // every (sequence, head) row block is contiguous and 16-byte aligned
      const uint8_t* kb = static_cast<const uint8_t*>(kv.k) + hr * kv.max_len * L::row;
      const uint8_t* vb = static_cast<const uint8_t*>(kv.v) + hr * kv.max_len * L::row;
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % NS;
        if (!mbar_wait(&empty[st], (static_cast<uint32_t>(c / NS) & 1u) ^ 1u, wait_ns)) {
          set_error(err, DEV_TIMEOUT_PRODUCER);
          break;
        }
        const int t0 = t_begin + c * T;
        const uint32_t bytes = static_cast<uint32_t>(min(T, t_end - t0)) * L::row;
        uint8_t* sb = ring + st * L::bytes;
        mbar_arrive_expect_tx(&full[st], 2 * bytes);
        bulk_g2s(sb, kb + static_cast<size_t>(t0) * L::row, bytes, &full[st]);
        bulk_g2s(sb + T * L::row, vb + static_cast<size_t>(t0) * L::row, bytes, &full[st]);
      }
      const uint64_t drain = wait_ns > 1000000000ull ? wait_ns : 1000000000ull;
      for (int c = max(0, n_chunks - NS); c < n_chunks; ++c)
        mbar_wait(&full[c % NS], static_cast<uint32_t>(c / NS) & 1u, drain);
    }
  } else {
    const int tk = lane >> 2, cq = lane & 3;
    float qf[DPL];
    const __half* qp = q + static_cast<size_t>(i) * ldq + j * D + cq * DPL;
#pragma unroll
    for (int e = 0; e < DPL; e += 2) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(qp + e));
      qf[e] = f.x;
      qf[e + 1] = f.y;
    }
    float m_run = -INFINITY, l_run = 0.f;
    float acc[DPV];
#pragma unroll
    for (int e = 0; e < DPV; ++e) acc[e] = 0.f;
    bool bad = false;
    for (int c = 0; c < n_chunks; ++c) {
      const int st = c % NS;
      if (!bad && !mbar_wait(&full[st], static_cast<uint32_t>(c / NS) & 1u, wait_ns)) {
        set_error(err, DEV_TIMEOUT_CONSUMER);
        bad = true;
      }
      const int nt = min(T, t_end - (t_begin + c * T));
      const __half* sk = reinterpret_cast<const __half*>(ring + st * L::bytes);
      const __half* sv = sk + T * D;
      const int wt0 = warp * TW;
      float sc[TW / 8];
      float mloc = -INFINITY;
#pragma unroll
      for (int u = 0; u < TW / 8; ++u) {
        const int tt = wt0 + u * 8 + tk;
        const bool valid = !bad && tt < nt;
        float partial = 0.f;
        if (valid) {
          const uint4* kr = reinterpret_cast<const uint4*>(sk + tt * D + cq * DPL);
#pragma unroll
          for (int v = 0; v < DPL / 8; ++v) {
            const uint4 w = kr[v];
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ww[e]));
              partial = fmaf(qf[8 * v + 2 * e], f.x, partial);
              partial = fmaf(qf[8 * v + 2 * e + 1], f.y, partial);
            }
          }
        }
        partial += __shfl_xor_sync(0xffffffffu, partial, 1);
        partial += __shfl_xor_sync(0xffffffffu, partial, 2);
        sc[u] = valid ? partial * inv_sqrt_d : -INFINITY;
        mloc = fmaxf(mloc, sc[u]);
      }
      const float m_c = warp_max(mloc);
      if (m_c != -INFINITY) {
        const float m_new = fmaxf(m_run, m_c);
        const float alpha = m_run == -INFINITY ? 0.f : __expf(m_run - m_new);
        float pr[TW / 8];
        float my_s = 0.f;
#pragma unroll
        for (int u = 0; u < TW / 8; ++u) {
          pr[u] = sc[u] == -INFINITY ? 0.f : __expf(sc[u] - m_new);
          if (cq == 0) my_s += pr[u];
        }
        const float s_c = warp_sum(my_s);
        float part_v[DPV];
#pragma unroll
        for (int e = 0; e < DPV; ++e) part_v[e] = 0.f;
#pragma unroll
        for (int u = 0; u < TW / 8; ++u) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float p = __shfl_sync(0xffffffffu, pr[u], 4 * k);
            const int tt = wt0 + u * 8 + k;
            if (tt < nt) {
              const __half* vr = sv + tt * D + lane * DPV;
#pragma unroll
              for (int e = 0; e < DPV; e += 2) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(vr + e));
                part_v[e] = fmaf(p, f.x, part_v[e]);
                part_v[e + 1] = fmaf(p, f.y, part_v[e + 1]);
              }
            }
          }
        }
#pragma unroll
        for (int e = 0; e < DPV; ++e) acc[e] = acc[e] * alpha + part_v[e];
        l_run = l_run * alpha + s_c;
        m_run = m_new;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    if (lane == 0) {
      cm[warp] = m_run;
      cl[warp] = l_run;
    }
#pragma unroll
    for (int e = 0; e < DPV; ++e) cacc[warp][lane * DPV + e] = acc[e];
  }
  __syncthreads();
  merge_and_store<D>(cm, cl, cacc, out, ldo, i, j, hr, z, part, ctr, &last_flag);
}

template <int D>
cudaError_t launch_f16(const __half* q, int ldq, const KvView& kv, int b, int heads, int len, __half* out, int ldo,
                       int splits, float* part, int* ctr, cudaStream_t s) {
  using L = F16Stage<D>;
  static cudaError_t attr = cudaFuncSetAttribute(attn_decode_f16_kernel<D>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, L::stages * L::bytes);
  if (attr != cudaSuccess) return attr;
  int span = (len + splits - 1) / splits;
  span = (span + L::T - 1) / L::T * L::T;
  const int S = (len + span - 1) / span;
  dim3 grid(heads, b, S);
  return launch_pdl(attn_decode_f16_kernel<D>, grid, dim3(kQ4Threads), L::stages * L::bytes, s, q, ldq, kv, heads,
                    len, out, ldo, 1.0f / sqrtf(static_cast<float>(D)), span, part, ctr, runtime().wait_limit_ns,
                    runtime().err);
}

}  // namespace

int attn_decode_splits(int b, int heads, int len) {
  const int units = b * heads;
  const int target = 3 * runtime().num_sms;  // three CTAs per SM
  if (units >= target) return 1;
  const int s = std::min(std::min(kMaxSplits, (target + units - 1) / units), (len + 2 * kChunk - 1) / (2 * kChunk));
  return std::max(1, s);
}

size_t attn_decode_partial_bytes(int b, int heads, int d) {
  // splits are used only while b * heads is under the target, so the partial
  // rows never exceed 2 * target of them
  const int units = b * heads;
  const int target = 3 * runtime().num_sms;
  const int rows = units >= target ? 0 : std::min(units * kMaxSplits, units + target);
  return static_cast<size_t>(rows) * (d + 2) * sizeof(float);
}

cudaError_t launch_attn_decode(const __half* q, int ldq, const KvView& kv, int b, int heads, int d,
                               int kv_bits, int len, __half* out, int ldo, float* part, int* ctr,
                               const AppendRow& app, cudaStream_t s) {
  if (b == 0) return cudaSuccess;
  const int splits = (part != nullptr && ctr != nullptr) ? attn_decode_splits(b, heads, len) : 1;
  if (kv_bits == 16)
    return d == 128 ? launch_f16<128>(q, ldq, kv, b, heads, len, out, ldo, splits, part, ctr, s)
                    : launch_f16<64>(q, ldq, kv, b, heads, len, out, ldo, splits, part, ctr, s);
  if (splits == 1)
    return d == 128 ? launch_q4_dense<128>(q, ldq, kv, b, heads, len, out, ldo, app, s)
                    : launch_q4_dense<64>(q, ldq, kv, b, heads, len, out, ldo, app, s);
  if (app.pos >= 0) {
    // the split kernel streams the cache with bulk copies: append first
    const cudaError_t e = launch_kv_append(app.k, app.v, app.ld, b, 1, heads, d, 4, kv, app.pos, s);
    if (e != cudaSuccess) return e;
  }
  return d == 128 ? launch_q4_split<128>(q, ldq, kv, b, heads, len, out, ldo, splits, part, ctr, s)
                  : launch_q4_split<64>(q, ldq, kv, b, heads, len, out, ldo, splits, part, ctr, s);
}

}  // namespace flexq

// Causal prefill attention on the fp16 Q/K/V of the pass:
//   x_out = softmax(x_Q x_K^T / sqrt(.)) x_V   (before W_O),
// FlexGen walk-through section "P/D阶段计算" (prefill), per head as in the
// survey notes' eq. (2), with the autoregressive (causal) mask: query i sees
// keys 0..i.  By default the pass's K and V are used as computed (the cache
// keeps their quantized copy for the decode steps); with the configuration's
// prefill_kv_cache the K/V tiles are read back from the cache as stored
// ("FlexGen研究学术报告" section 三(C): compressed cache, dequantized before
// compute): fp16 rows of an fp16 cache, or 4-bit codes dequantized tile by tile
// into shared memory (fp16(fp32(code * scale) + min), the codec's rounding).
//
// Flash-attention style: one CTA = 64 queries of one (sequence, head), 4 warps
// x 16 query rows; K/V tiles of 64 keys double-buffered in shared memory with
// cp.async; Q K^T and P V on mma.sync m16n8k16 (fp16 in, fp32 accumulate);
// online softmax in registers with base-2 exponentials.  Prefill attention is
// a few percent of the prefill FLOPs (2 b s^2 h against 24 b s h^2), so the
// legacy warp-level MMA is enough here.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace flexq {
namespace {

constexpr int BQ = 64;
constexpr int BK = 64;
constexpr int kThreads = 128;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Byte offset of 16-byte chunk `ch` of row `r` in a [rows][D] fp16 tile with
// the chunk index XOR-swizzled by the row (conflict-free ldmatrix).
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int ch) {
  return static_cast<uint32_t>(r * (D * 2) + ((ch ^ (r & 7)) * 16));
}

template <int D>
__device__ __forceinline__ void load_tile(uint32_t sbase, const __half* g, int ld, int row0, int rows_valid) {
  constexpr int CH = D / 8;
  for (int idx = threadIdx.x; idx < 64 * CH; idx += kThreads) {
    const int r = idx / CH, ch = idx % CH;
    const bool valid = r < rows_valid;
    const __half* src = g + static_cast<size_t>(valid ? row0 + r : row0) * ld + ch * 8;
    cp_async16(sbase + swz<D>(r, ch), src, valid);
  }
}

// 4-bit cache tile of keys k0 .. k0 + 63 (cache slots pos0 + k0 ..) of head
// row hr, dequantized into the swizzled [64][D] fp16 layout; rows past
// `rows_valid` are zero.  K: one (key, 64-element group) per thread step;
// V (token-interleaved words): one (8-token block, 8 dimensions) per step,
// written as 8 rows of one 16-byte chunk.
__device__ __forceinline__ __half dq16(uint32_t code, float sc, float mn) {
  return __float2half_rn(__fadd_rn(__fmul_rn(static_cast<float>(code), sc), mn));
}

template <int D>
__device__ __forceinline__ void load_tile_q4(uint32_t sK, uint32_t sV, const KvView& kv, size_t hr, int pos0, int k0,
                                             int rows_valid) {
  constexpr int G = D / 64;
  const uint8_t* kc = static_cast<const uint8_t*>(kv.k) + (hr * kv.max_len + pos0 + k0) * (D / 2);
  const __half2* km = static_cast<const __half2*>(kv.k_meta) + (hr * kv.max_len + pos0 + k0) * G;
  const __half2* vm = static_cast<const __half2*>(kv.v_meta) + (hr * kv.max_len + pos0 + k0) * G;
  const uint32_t* vw = static_cast<const uint32_t*>(kv.v) + (hr * (kv_pad_len(kv.max_len) / 8) + (pos0 + k0) / 8) * D;
  for (int idx = threadIdx.x; idx < 64 * G; idx += kThreads) {
    const int r = idx / G, gg = idx % G;
    uint4 out[8];
    if (r < rows_valid) {
      const uint4 c0 = *reinterpret_cast<const uint4*>(kc + r * (D / 2) + gg * 32);
      const uint4 c1 = *reinterpret_cast<const uint4*>(kc + r * (D / 2) + gg * 32 + 16);
      const float2 ms = __half22float2(km[r * G + gg]);
      const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        __half e[8];
#pragma unroll
        for (int n = 0; n < 8; ++n) e[n] = dq16((w[c] >> (4 * n)) & 0xFu, ms.y, ms.x);
        out[c] = *reinterpret_cast<const uint4*>(e);
      }
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) out[c] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c)
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sK + swz<D>(r, gg * 8 + c)), "r"(out[c].x),
                   "r"(out[c].y), "r"(out[c].z), "r"(out[c].w)
                   : "memory");
  }
  for (int idx = threadIdx.x; idx < 8 * (D / 8); idx += kThreads) {
    const int bi = idx / (D / 8), dc = idx % (D / 8);
    const int gg = (dc * 8) / 64;
    uint32_t w[8];
    const bool any = bi * 8 < rows_valid;
    if (any) {
      const uint4 a = *reinterpret_cast<const uint4*>(vw + bi * D + dc * 8);
      const uint4 b = *reinterpret_cast<const uint4*>(vw + bi * D + dc * 8 + 4);
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int r = bi * 8 + kk;
      uint4 o4 = make_uint4(0u, 0u, 0u, 0u);
      if (r < rows_valid) {
        const float2 ms = __half22float2(vm[r * G + gg]);
        __half e[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) e[c] = dq16((w[c] >> (4 * kk)) & 0xFu, ms.y, ms.x);
        o4 = *reinterpret_cast<const uint4*>(e);
      }
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sV + swz<D>(r, dc)), "r"(o4.x), "r"(o4.y),
                   "r"(o4.z), "r"(o4.w)
                   : "memory");
    }
  }
}

// K/V source: kPass = the pass's rows in the Q/K/V buffer; kCache16 / kCache4
// = the layer's cache (slots pos0 ..).
enum PrefillKv : int { kPass = 0, kCache16 = 1, kCache4 = 2 };

struct PrefillArgs {
  const __half* q;  // row (sequence i, token t) at q + (i * seq + t) * ldq, head j at + j * D
  int ldq;
  const __half* k;  // kPass: K / V columns of the same buffer (ld = ldkv)
  const __half* v;
  int ldkv;
  KvView kv;        // kCache16 / kCache4
  int pos0;         // first cache slot of the pass (a multiple of 8 for kCache4)
  int seq, heads;
  __half* out;
  int ldo;
  float scale_log2;
};

template <int D, int KV>
__global__ void __launch_bounds__(kThreads) attn_prefill_kernel(const PrefillArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + BQ * D * 2;
  const uint32_t sV = sK + 2 * BK * D * 2;
  const int qb = gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int j = blockIdx.y, i = blockIdx.z;
  const int seq = a.seq;
  const size_t hr = static_cast<size_t>(i) * a.heads + j;
  const __half* gQ = a.q + static_cast<size_t>(i) * seq * a.ldq + j * D;
  const __half* gK;
  const __half* gV;
  int ldkv;
  if (KV == kPass) {
    gK = a.k + static_cast<size_t>(i) * seq * a.ldkv + j * D;
    gV = a.v + static_cast<size_t>(i) * seq * a.ldkv + j * D;
    ldkv = a.ldkv;
  } else {
    gK = static_cast<const __half*>(a.kv.k) + (hr * a.kv.max_len + a.pos0) * D;
    gV = static_cast<const __half*>(a.kv.v) + (hr * a.kv.max_len + a.pos0) * D;
    ldkv = D;
  }
  __half* out = a.out;
  const int ldo = a.ldo;
  const float scale_log2 = a.scale_log2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = qb * BQ;

  load_tile<D>(sQ, gQ, a.ldq, q0, min(BQ, seq - q0));
  if (KV == kCache4) {
    load_tile_q4<D>(sK, sV, a.kv, hr, a.pos0, 0, min(BK, seq));
  } else {
    load_tile<D>(sK, gK, ldkv, 0, min(BK, seq));
    load_tile<D>(sV, gV, ldkv, 0, min(BK, seq));
  }
  cp_commit();

  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const int g = lane >> 2, c = lane & 3;
  const int qrow0 = q0 + warp * 16 + g;  // rows qrow0 and qrow0 + 8
  const int ntiles = qb + 1;

  for (int kt = 0; kt < ntiles; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < ntiles) {
      const int k0 = (kt + 1) * BK;
      if (KV == kCache4) {
        load_tile_q4<D>(sK + (buf ^ 1) * BK * D * 2, sV + (buf ^ 1) * BK * D * 2, a.kv, hr, a.pos0, k0,
                        min(BK, seq - k0));
      } else {
        load_tile<D>(sK + (buf ^ 1) * BK * D * 2, gK, ldkv, k0, min(BK, seq - k0));
        load_tile<D>(sV + (buf ^ 1) * BK * D * 2, gV, ldkv, k0, min(BK, seq - k0));
      }
    }
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    const uint32_t kbase = sK + buf * BK * D * 2;
    const uint32_t vbase = sV + buf * BK * D * 2;

    float s[BK / 8][4];
#pragma unroll
    for (int n = 0; n < BK / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(sQ + swz<D>(warp * 16 + (lane & 15), kk * 2 + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
      for (int nb = 0; nb < BK / 16; ++nb) {
        const int mi = lane >> 3;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbase + swz<D>(nb * 16 + (mi >> 1) * 8 + (lane & 7), kk * 2 + (mi & 1)), b0, b1, b2, b3);
        mma16816(s[2 * nb], a0, a1, a2, a3, b0, b1);
        mma16816(s[2 * nb + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    // causal mask on the diagonal tile, then online softmax
    const bool diag = kt == qb;
    float mnew[2] = {m_r[0], m_r[1]};
#pragma unroll
    for (int n = 0; n < BK / 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kt * BK + n * 8 + 2 * c + (e & 1);
        const int qrow = qrow0 + (e >> 1) * 8;
        float v = s[n][e] * scale_log2;
        if (diag && key > qrow) v = -INFINITY;
        s[n][e] = v;
        mnew[e >> 1] = fmaxf(mnew[e >> 1], v);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mnew[r] = fmaxf(mnew[r], __shfl_xor_sync(0xffffffffu, mnew[r], 1));
      mnew[r] = fmaxf(mnew[r], __shfl_xor_sync(0xffffffffu, mnew[r], 2));
    }
    float alpha[2], rs[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 2; ++r) alpha[r] = exp2f(m_r[r] - mnew[r]);
#pragma unroll
    for (int n = 0; n < BK / 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[n][e] - mnew[e >> 1]);
        s[n][e] = p;
        rs[e >> 1] += p;
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 1);
      rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 2);
      l_r[r] = l_r[r] * alpha[r] + rs[r];
      m_r[r] = mnew[r];
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      o[n][0] *= alpha[0];
      o[n][1] *= alpha[0];
      o[n][2] *= alpha[1];
      o[n][3] *= alpha[1];
    }
    // O += P V
#pragma unroll
    for (int t = 0; t < BK / 16; ++t) {
      const uint32_t a0 = pack_h2(s[2 * t][0], s[2 * t][1]);
      const uint32_t a1 = pack_h2(s[2 * t][2], s[2 * t][3]);
      const uint32_t a2 = pack_h2(s[2 * t + 1][0], s[2 * t + 1][1]);
      const uint32_t a3 = pack_h2(s[2 * t + 1][2], s[2 * t + 1][3]);
#pragma unroll
      for (int nb = 0; nb < D / 16; ++nb) {
        const int mi = lane >> 3;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbase + swz<D>(t * 16 + (mi & 1) * 8 + (lane & 7), nb * 2 + (mi >> 1)), b0, b1, b2, b3);
        mma16816(o[2 * nb], a0, a1, a2, a3, b0, b1);
        mma16816(o[2 * nb + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();
  }
  // normalise and store
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qrow = qrow0 + r * 8;
    if (qrow >= seq) continue;
    const float inv = 1.0f / l_r[r];
    __half* dst = out + (static_cast<size_t>(i) * seq + qrow) * ldo + j * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
      *reinterpret_cast<__half2*>(dst + n * 8 + 2 * c) =
          __floats2half2_rn(o[n][2 * r] * inv, o[n][2 * r + 1] * inv);
  }
}

template <int D, int KV>
cudaError_t launch_d(PrefillArgs a, int b, cudaStream_t s) {
  const int smem = (BQ + 4 * BK) * D * 2;
  static const cudaError_t configured =
      cudaFuncSetAttribute(attn_prefill_kernel<D, KV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (configured != cudaSuccess) return configured;
  dim3 grid((a.seq + BQ - 1) / BQ, a.heads, b);
  a.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  attn_prefill_kernel<D, KV><<<grid, kThreads, smem, s>>>(a);
  return launched();
}

template <int KV>
cudaError_t launch_kv(const PrefillArgs& a, int b, int d, cudaStream_t s) {
  return d == 128 ? launch_d<128, KV>(a, b, s) : launch_d<64, KV>(a, b, s);
}

}  // namespace

cudaError_t launch_attn_prefill(const __half* qkv, int ldqkv, int b, int seq, int heads, int d, __half* out,
                                int ldo, cudaStream_t s) {
  if (b == 0 || seq == 0) return cudaSuccess;
  PrefillArgs a{};
  a.q = qkv;
  a.ldq = ldqkv;
  a.k = qkv + heads * d;
  a.v = qkv + 2 * heads * d;
  a.ldkv = ldqkv;
  a.seq = seq;
  a.heads = heads;
  a.out = out;
  a.ldo = ldo;
  return launch_kv<kPass>(a, b, d, s);
}

cudaError_t launch_attn_prefill_cache(const __half* q, int ldq, const KvView& kv, int kv_bits, int pos0, int b,
                                      int seq, int heads, int d, __half* out, int ldo, cudaStream_t s) {
  if (b == 0 || seq == 0) return cudaSuccess;
  if (kv_bits == 4 && pos0 % 8 != 0) return cudaErrorInvalidValue;
  PrefillArgs a{};
  a.q = q;
  a.ldq = ldq;
  a.kv = kv;
  a.pos0 = pos0;
  a.seq = seq;
  a.heads = heads;
  a.out = out;
  a.ldo = ldo;
  return kv_bits == 4 ? launch_kv<kCache4>(a, b, d, s) : launch_kv<kCache16>(a, b, d, s);
}

}  // namespace flexq

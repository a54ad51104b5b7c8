// Dequant-fused linear layers on the 5th-generation tensor core.
//
//   Y[m][n] = epilogue( X[m][k] . W_hat[n][k]^T )
//
// W_hat is the group-wise 4-bit weight ("FlexGen研究学术报告", section 三(C):
// groups of 64 contiguous elements along K_in, fp16 min/scale, dequantized to
// fp16 before compute) or a plain fp16 weight.  The layers are x W_Q/K/V,
// (.) W_O + x, f_gelu(x_out W_1) and (.) W_2 + x_out of the FlexGen
// walk-through (section "P/D阶段计算"), with the [h] / [ih] biases of section
// "内存占用分析" fused into the epilogue.
//
// One output tile = 128 features x up to 256 tokens; the weight is the MMA's A
// operand, so a small decode batch becomes the MMA's N.  A persistent CTA per
// SM walks a list of (tile, k-block range) segments in k-steps of KS 64-wide
// k-blocks:
//   warp 0      weight producer: per k-step one cp.async.bulk of the KS packed
//               chunks (codes + min/scale, 4608 contiguous bytes per k-block),
//               or one 3-D tensor box of fp16 weights;
//   warp 14     activation producer: per k-step one 3-D tensor box {64 columns,
//               tokens, KS k-blocks}, i.e. KS 128-byte-swizzled tiles;
//   warps 2-9   dequantize the weight rows ((code | 0x6400) is the fp16 value
//               1024 + code; one half2 subtract and one half2 fused multiply-
//               add give code * scale + min rounded once): decode-sized tiles
//               into tensor memory (tcgen05.st, one weight row per TMEM lane),
//               larger tiles into a shared-memory ring in the UMMA K-major
//               SW128 layout;
//   warp 1      owns TMEM and, from one thread, issues tcgen05.mma.kind::f16
//               (M=128, N=tokens, K=16; A from tensor or shared memory, B from
//               shared memory);
//   warps 10-13 epilogue (below).
// A copying thread completes about one copy per memory round trip whatever
// its size (up to ~16 KB), so each ring has its own thread and every copy
// moves a whole k-step: KS = 4 for 4-bit decode tiles of <= 128 tokens, 2 for
// other decode tiles, 1 for prefill tiles.
//
// Epilogue (warps 10-13, one TMEM lane quarter each): tcgen05.ld, + bias,
// GELU, + residual, fp16 or fp32 store; two accumulator buffers let it overlap
// the next segment's main loop.
// Scheduling: whole tiles round-robin over the SMs when there are many; when
// the grid is small (decode), each SM takes an equal share of all k-blocks
// (stream-K), so tiles may be split across CTAs.  Every contributor of a split
// tile counts itself in; the one that arrives last does not write its own
// partial: it waits until the others' fp32 partials are published, then sums
// them and its own accumulator (in TMEM) in contributor order and applies the
// epilogue, so results do not depend on timing.
// Every wait is bounded; on expiry the CTA records an error code in the device
// error word and unwinds (no trap).
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace flexq {
namespace {

constexpr int kThreads = 512;  // 16 warps: W producer, MMA, 8 dequantizing, 4 epilogue, B producer, MMA
constexpr int kDequantThreads = 256;
constexpr int kEpiThreads = 128;
constexpr int kEpiWarp0 = 10;
constexpr int kBWarp = 14;
constexpr int kMmaWarp2 = 15;  // second MMA-issuing warp (issuer 0 is warp 1)
constexpr int kATileBytes = 128 * 64 * 2;
constexpr int kMaxSmem = 227 * 1024;
constexpr int kBarrierBytes = 1024;  // mbarriers, TMEM address, flags, finalize slot list
constexpr int kMaxBarriers = 56;     // mbarriers fit in the first 448 bytes of that region
constexpr int kEpiStageBytes = 4 * 16 * 33 * 4;  // per epilogue warp: 16 tokens x 33 floats
constexpr int kMaxWStages = 16;
constexpr int kMinItersPerCta = 8;
constexpr int kMaxContrib = 64;
constexpr int kDecodeMaxTok = 160;

enum SchedMode : int { SCHED_TILES = 0, SCHED_STREAMK = 1, SCHED_SPLITS = 2 };

struct Sched {
  int mode;
  int grid;
  int tiles;        // n_tiles * tok_tiles
  int n_tiles;
  int kb_total;     // k-blocks per tile
  long long iters;  // tiles * kb_total
  int splits, per;  // SCHED_SPLITS
};

struct GemmParams {
  const uint8_t* wq;
  int m, n, k;
  int tok_tile;
  int kb_real;  // 64-wide k-blocks of K
  int w_stages, b_stages, a_stages;     // ring depths: weights, activations, dequantized A
  uint32_t w_slot_bytes, b_slot_bytes;
  uint32_t acc_cols;    // TMEM columns between accumulator buffers
  uint32_t chain_cols;  // TMEM columns between the issuers' accumulators of a buffer
  int issuers;          // MMA-issuing threads, 1, 2 or 4 (k-blocks of a step round-robin)
  int acc_bufs;         // accumulator buffers (2: the epilogue overlaps the next segment)
  uint32_t tmem_alloc;  // columns allocated (power of two)
  uint32_t a_col0;      // first TMEM column of the dequantized A ring (A in tensor memory)
  Sched sc;
  const __half* bias;
  const __half* residual;
  int ld_res;
  __half* y;
  int ldy;
  float* yf;
  int ldyf;
  int epi;
  float* partials;  // [slot][tok_tile][128]
  int* counters;    // [tiles][2]: contributors arrived, partials published
  uint64_t wait_ns;
  uint32_t* err;
  int kv_on;        // decode QKV: K/V tiles go to the fp16 cache
  KvFuse kv;
  int ln_on;        // decode out-proj / FC2: LayerNorm of the rows after a grid barrier
  LnFuse ln;
};

struct Seg {
  int tile, kb0, kb1;
  bool full;
  int slot;
};

// Position and phase parity in a ring of mbarrier-guarded slots, advanced
// without divisions (the role threads are latency-bound scalar loops).
struct Ring {
  int s = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void next(int n) {
    if (++s == n) {
      s = 0;
      ph ^= 1u;
    }
  }
};

__device__ __forceinline__ long long sk_start(const Sched& s, int c) {
  return static_cast<long long>(c) * s.iters / s.grid;
}

// Segment q of CTA c; false when the CTA has no more work.
__device__ __forceinline__ bool get_seg(const Sched& s, int c, int q, Seg& g) {
  if (s.mode == SCHED_TILES) {
    const long long t = c + static_cast<long long>(q) * s.grid;
    if (t >= s.tiles) return false;
    g.tile = static_cast<int>(t);
    g.kb0 = 0;
    g.kb1 = s.kb_total;
    g.full = true;
    g.slot = -1;
    return true;
  }
  if (s.mode == SCHED_SPLITS) {
    if (q > 0) return false;
    g.tile = c / s.splits;
    const int part = c % s.splits;
    g.kb0 = part * s.per;
    g.kb1 = min(s.kb_total, g.kb0 + s.per);
    g.full = s.splits == 1;
    g.slot = c;
    return g.kb1 > g.kb0;
  }
  // The CTA's iterations [it0, it1) touch tiles t0 .. t1; its first and last
  // tiles may be partial (shared with the neighbouring CTAs).  Partial
  // segments run first, then the whole tiles: a split tile's contributors
  // then all finish it early, its fixup overlaps the whole tiles, and the
  // kernel ends on plain epilogues rather than on waits for partners.
  const long long it0 = sk_start(s, c), it1 = sk_start(s, c + 1);
  if (it1 <= it0) return false;
  const long long t0 = it0 / s.kb_total, t1 = (it1 - 1) / s.kb_total;
  const int n_seg = static_cast<int>(t1 - t0 + 1);
  if (q >= n_seg) return false;
  const bool last_part = it1 % s.kb_total != 0 && n_seg > 1;
  const int i = !last_part ? q : q == 0 ? n_seg - 1 : q - 1;  // index in iteration order
  const long long it = i == 0 ? it0 : (t0 + i) * s.kb_total;
  g.tile = static_cast<int>(t0 + i);
  g.kb0 = static_cast<int>(it - static_cast<long long>(g.tile) * s.kb_total);
  const long long end = min(it1, static_cast<long long>(g.tile + 1) * s.kb_total);
  g.kb1 = static_cast<int>(end - static_cast<long long>(g.tile) * s.kb_total);
  g.full = g.kb0 == 0 && g.kb1 == s.kb_total;
  g.slot = 2 * c + (i == 0 ? 0 : 1);
  return true;
}

// First CTA whose stream-K range reaches into the iterations starting at t0.
__device__ __forceinline__ int sk_first_contributor(const Sched& s, long long t0) {
  int lo = static_cast<int>(t0 * s.grid / s.iters);
  while (lo > 0 && sk_start(s, lo) > t0) --lo;
  while (lo + 1 < s.grid && sk_start(s, lo + 1) <= t0) ++lo;
  return lo;
}

__device__ __forceinline__ uint64_t drain_ns(uint64_t wait_ns) {
  return wait_ns > 1000000000ull ? wait_ns : 1000000000ull;
}

__device__ __forceinline__ float gelu_erf(float v) {
  return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}

__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// 8 codes (tiled nibble order) -> 8 fp16 values code * s + m.
__device__ __forceinline__ uint4 dequant8(uint32_t w, __half2 s2, __half2 m2) {
  const __half2 k1024 = __float2half2_rn(1024.0f);
  uint4 r;
  r.x = h2_as_u32(__hfma2(__hsub2(u32_as_h2((w & 0x000F000Fu) | 0x64006400u), k1024), s2, m2));
  r.y = h2_as_u32(__hfma2(__hsub2(u32_as_h2(((w >> 4) & 0x000F000Fu) | 0x64006400u), k1024), s2, m2));
  r.z = h2_as_u32(__hfma2(__hsub2(u32_as_h2(((w >> 8) & 0x000F000Fu) | 0x64006400u), k1024), s2, m2));
  r.w = h2_as_u32(__hfma2(__hsub2(u32_as_h2(((w >> 12) & 0x000F000Fu) | 0x64006400u), k1024), s2, m2));
  return r;
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); }

// Named barrier over kCount threads that also ORs a predicate across them, so
// a branch taken on the result is uniform (no thread skips a later barrier).
template <int kCount>
__device__ __forceinline__ bool bar_any(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "n"(kCount)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ bool al16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

__device__ __forceinline__ void load_h16(const __half* src, int count, float (&v)[16]) {
  if (count == 16 && al16(src)) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(src));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(src) + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float2 f = __half22float2(u32_as_h2(w[u]));
      v[2 * u] = f.x;
      v[2 * u + 1] = f.y;
    }
  } else {
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = u < count ? __half2float(src[u]) : 0.f;
  }
}

// Bias of output features f0..f0+15 (zero where the epilogue adds none).
__device__ __forceinline__ void load_bias16(const GemmParams& p, int f0, float (&bv)[16]) {
  if ((p.epi & EPI_BIAS) && !(p.epi & EPI_F32_OUT) && f0 < p.n) {
    load_h16(p.bias + f0, min(16, p.n - f0), bv);
  } else {
#pragma unroll
    for (int u = 0; u < 16; ++u) bv[u] = 0.f;
  }
}

// Epilogue for 16 consecutive output features f0..f0+15 of one token; bv holds
// their bias.  Every load is issued before any store, and full aligned rows
// use 16-byte vectors.
__device__ __forceinline__ void store_row16(const GemmParams& p, float (&v)[16], const float (&bv)[16], int tok,
                                            int f0) {
  const int count = min(16, p.n - f0);
  if (p.epi & EPI_F32_OUT) {
    float* dst = p.yf + static_cast<size_t>(tok) * p.ldyf + f0;
    if (count == 16 && al16(dst)) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        reinterpret_cast<float4*>(dst)[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
    } else {
      for (int u = 0; u < count; ++u) dst[u] = v[u];
    }
    return;
  }
  float rv[16];
  if (p.epi & EPI_RESIDUAL) {
    load_h16(p.residual + static_cast<size_t>(tok) * p.ld_res + f0, count, rv);
  } else {
#pragma unroll
    for (int u = 0; u < 16; ++u) rv[u] = 0.f;
  }
  uint32_t packed[8];
#pragma unroll
  for (int u = 0; u < 16; u += 2) {
    float a = v[u] + bv[u], b = v[u + 1] + bv[u + 1];
    if (p.epi & EPI_GELU) {
      a = gelu_erf(a);
      b = gelu_erf(b);
    }
    packed[u / 2] = h2_as_u32(__floats2half2_rn(a + rv[u], b + rv[u + 1]));
  }
  __half* dst = p.y + static_cast<size_t>(tok) * p.ldy + f0;
  if (count == 16 && al16(dst)) {
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  } else {
#pragma unroll
    for (int u = 0; u < 16; u += 2) {
      if (u < count) dst[u] = __low2half(u32_as_h2(packed[u / 2]));
      if (u + 1 < count) dst[u + 1] = __high2half(u32_as_h2(packed[u / 2]));
    }
  }
}

// Accumulator buffer and phase parity used by segment q.
__device__ __forceinline__ void acc_slot(int q, int bufs, int& buf, uint32_t& parity) {
  if (bufs == 2) {
    buf = q & 1;
    parity = static_cast<uint32_t>(q >> 1) & 1u;
  } else {
    buf = 0;
    parity = static_cast<uint32_t>(q) & 1u;
  }
}

// Shared-memory words of the epilogue and the teardown, after the rings.
struct Ctl {
  uint64_t* accf;  // [2] accumulator buffer complete
  uint64_t* acce;  // [2] accumulator buffer drained
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  volatile int* last_flag;
  volatile int* fin_count;
  volatile int* fin_me;
  int* fin_slots;  // [kMaxContrib]
  float* stage;    // [4][16][33]
};

__device__ __forceinline__ Ctl make_ctl(uint8_t* region, uint64_t* accf) {
  Ctl c;
  c.accf = accf;
  c.acce = accf + 2;
  c.tmem_slot = reinterpret_cast<uint32_t*>(region + 8 * kMaxBarriers);
  c.abort_flag = reinterpret_cast<volatile int*>(c.tmem_slot + 1);
  c.last_flag = c.abort_flag + 1;
  c.fin_count = c.abort_flag + 2;
  c.fin_me = c.abort_flag + 3;
  c.fin_slots = reinterpret_cast<int*>(region + kBarrierBytes / 2);
  c.stage = reinterpret_cast<float*>(region + kBarrierBytes);
  return c;
}

// Bounded wait until a global counter reaches `target` (the other
// contributors of a split tile have published their partials).
__device__ __forceinline__ bool wait_counter(const int* ctr, int target, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
    __nanosleep(64);
  }
}

// ---------------------------------------------------------------------------
// epilogue role (warps kEpiWarp0 .. kEpiWarp0 + 3)
// ---------------------------------------------------------------------------
// 16 accumulator columns (tokens col .. col + 15) of this thread's TMEM lane:
// the sum of the issuers' accumulators, in issuer order.  Warp-wide.
__device__ __forceinline__ void acc_load16(const GemmParams& p, uint32_t tbase, uint32_t col, float (&v)[16]) {
  uint32_t rr[16];
  __syncwarp();
  tmem_ld_x16(tbase + col, rr);
  tmem_ld_wait();
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(rr[j]);
  if (p.issuers > 1) {
    __syncwarp();
    tmem_ld_x16(tbase + p.chain_cols + col, rr);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] += __uint_as_float(rr[j]);
  }
}

__device__ void epilogue_role(const GemmParams& p, const Ctl& c, uint32_t tmem_base, int warp, int lane) {
  pdl_wait();  // the residual, outputs, partials and counters belong to the stream's order
  const Sched& sc = p.sc;
  const int cta = blockIdx.x;
  const int et = threadIdx.x - kEpiWarp0 * 32;
  const int qd = warp & 3;          // TMEM lane quarter this warp may access
  const int frow = qd * 32 + lane;  // feature row of the tile this thread reads from TMEM
  const int jt = lane >> 1, hf = lane & 1;
  float* stg = c.stage + (warp - kEpiWarp0) * 16 * 33;
  Seg g;
  for (int q = 0; get_seg(sc, cta, q, g); ++q) {
    int buf;
    uint32_t par;
    acc_slot(q, p.acc_bufs, buf, par);
    const bool ok = mbar_wait(&c.accf[buf], par, drain_ns(p.wait_ns));
    if (!ok) set_error(p.err, DEV_TIMEOUT_EPILOGUE);
    tc_fence_after();
    const bool aborted = bar_any<kEpiThreads>(1, !ok || *c.abort_flag);
    if (aborted) {
      tc_fence_before();
      mbar_arrive(&c.acce[buf]);
      continue;
    }
    const int n_tile = g.tile % sc.n_tiles;
    const int tok0 = (g.tile / sc.n_tiles) * p.tok_tile;
    const uint32_t tbase =
        tmem_base + static_cast<uint32_t>(buf) * p.acc_cols + (static_cast<uint32_t>(qd * 32) << 16);
    const int f_out = n_tile * 128 + qd * 32 + hf * 16;  // features this lane finishes
    // decode QKV with an fp16 cache: the K and V tiles go to the cache slot
    const bool kv_tile = p.kv_on && n_tile * 128 >= p.kv.h;
    // Split tile: count in; the last to arrive finishes the tile.
    int ns = 1, me = 0;
    if (!g.full) {
      if (et == 0) {
        int n = 0, mine = 0;
        if (sc.mode == SCHED_SPLITS) {
          for (int part = 0; part < sc.splits && n < kMaxContrib; ++part) {
            if (g.tile * sc.splits + part == g.slot) mine = n;
            c.fin_slots[n++] = g.tile * sc.splits + part;
          }
        } else {
          const long long t0 = static_cast<long long>(g.tile) * sc.kb_total;
          for (int cc = sk_first_contributor(sc, t0);
               cc < sc.grid && sk_start(sc, cc) < t0 + sc.kb_total && n < kMaxContrib; ++cc) {
            const int sl = 2 * cc + (sk_start(sc, cc) >= t0 ? 0 : 1);
            if (sl == g.slot) mine = n;
            c.fin_slots[n++] = sl;
          }
        }
        *c.fin_count = n;
        *c.fin_me = mine;
        const int old = atomicAdd(&p.counters[2 * g.tile], 1);
        *c.last_flag = old == n - 1;
      }
      epi_bar();
      const bool last = *c.last_flag;
      ns = *c.fin_count;
      me = *c.fin_me;
      if (!last) {
        // publish this contributor's fp32 partial (a warp stores 32
        // consecutive features of one token)
        float* slot = p.partials + static_cast<size_t>(g.slot) * p.tok_tile * 128;
        for (int c0 = 0; c0 < p.tok_tile; c0 += 16) {
          float a[16];
          acc_load16(p, tbase, static_cast<uint32_t>(c0), a);
#pragma unroll
          for (int j = 0; j < 16; ++j) __stcg(slot + (c0 + j) * 128 + frow, a[j]);
        }
        tc_fence_before();
        mbar_arrive(&c.acce[buf]);
        __threadfence();
        epi_bar();
        if (et == 0) atomicAdd(&p.counters[2 * g.tile + 1], 1);
        continue;
      }
      if (et == 0 && !wait_counter(&p.counters[2 * g.tile + 1], ns - 1, drain_ns(p.wait_ns)))
        set_error(p.err, DEV_TIMEOUT_EPILOGUE);
      epi_bar();
    }
    // Finish the tile: the accumulator (plus the other contributors' partials,
    // summed in contributor order), then bias / GELU / residual.
    float bv[16];
    load_bias16(p, f_out, bv);
    const bool one_other = !g.full && ns == 2;
    const float* other =
        one_other ? p.partials + static_cast<size_t>(c.fin_slots[1 - me]) * p.tok_tile * 128 : nullptr;
    float nxt[16];  // the other contributor's values for the next 16 tokens
    if (one_other) {
#pragma unroll
      for (int j = 0; j < 16; ++j) nxt[j] = __ldcg(other + j * 128 + frow);
    }
    for (int c0 = 0; c0 < p.tok_tile; c0 += 16) {
      float acc[16];
      float v[16];
      if (one_other) {
        float cur[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) cur[j] = nxt[j];
        if (c0 + 16 < p.tok_tile) {
#pragma unroll
          for (int j = 0; j < 16; ++j) nxt[j] = __ldcg(other + (c0 + 16 + j) * 128 + frow);
        }
        acc_load16(p, tbase, static_cast<uint32_t>(c0), acc);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = me == 0 ? (0.f + acc[j]) + cur[j] : (0.f + cur[j]) + acc[j];
      } else if (!g.full) {
        acc_load16(p, tbase, static_cast<uint32_t>(c0), acc);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.f;
        for (int k = 0; k < ns; ++k) {
          if (k == me) {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] += acc[j];
          } else {
            const float* src = p.partials + static_cast<size_t>(c.fin_slots[k]) * p.tok_tile * 128;
            float t[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) t[j] = __ldcg(src + (c0 + j) * 128 + frow);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] += t[j];
          }
        }
      } else {
        acc_load16(p, tbase, static_cast<uint32_t>(c0), v);
      }
      // transpose 32 features x 16 tokens through shared memory so each lane
      // finishes 16 consecutive features of one token
#pragma unroll
      for (int j = 0; j < 16; ++j) stg[j * 33 + lane] = v[j];
      __syncwarp();
      const int tok = tok0 + c0 + jt;
      if (kv_tile) {
        // this lane's 16 features of its token (+ bias) go to slot pos
        if (tok < p.m) {
          uint32_t packed[8];
#pragma unroll
          for (int u = 0; u < 16; u += 2)
            packed[u / 2] = h2_as_u32(__floats2half2_rn(stg[jt * 33 + hf * 16 + u] + bv[u],
                                                        stg[jt * 33 + hf * 16 + u + 1] + bv[u + 1]));
          const bool is_v = f_out >= 2 * p.kv.h;
          const int cc = f_out - (is_v ? 2 * p.kv.h : p.kv.h);
          uint4* dst = reinterpret_cast<uint4*>(
              (is_v ? p.kv.v : p.kv.k) +
              ((static_cast<size_t>(tok) * p.kv.heads + cc / p.kv.d) * p.kv.max_len + p.kv.pos) * p.kv.d + cc % p.kv.d);
          dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
      } else if (tok < p.m && f_out < p.n) {
        float o[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) o[u] = stg[jt * 33 + hf * 16 + u];
        store_row16(p, o, bv, tok, f_out);
      }
      __syncwarp();
    }
    // A split tile's counters go back to zero once it is finished (every
    // contributor has counted in and published), so a sequence of launches
    // needs them zeroed only once.
    if (!g.full && et == 0) {
      p.counters[2 * g.tile] = 0;
      p.counters[2 * g.tile + 1] = 0;
    }
    tc_fence_before();
    mbar_arrive(&c.acce[buf]);
  }
}

// Grid-wide barrier of a cooperative launch, entered by one thread per CTA
// after its CTA's stores are complete.  sync[0] counts arrivals, sync[1] is
// the generation: the last arrival resets the count and advances the
// generation, the others wait (bounded) for the generation to move.  Both
// words return to their entry values' pattern (count 0), so one zeroing
// serves every later launch.
__device__ __forceinline__ bool grid_sync(int* sync, int nblocks, uint64_t limit_ns) {
  int g0;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(g0) : "l"(sync + 1) : "memory");
  __threadfence();
  const int old = atomicAdd(sync, 1);
  if (old == nblocks - 1) {
    atomicExch(sync, 0);
    __threadfence();
    atomicAdd(sync + 1, 1);
    return true;
  }
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    int g;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(g) : "l"(sync + 1) : "memory");
    if (g != g0) break;
    if (globaltimer_ns() - t0 > limit_ns) return false;
    __nanosleep(32);
  }
  __threadfence();
  return true;
}

__device__ __forceinline__ float block_sum_all(float v, float* red) {
  v = warp_sum(v);
  __syncthreads();
  if (lane_id() == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) r += red[w];
  return r;
}

// LayerNorm phase of the fused out-proj / FC2 (after every CTA's tiles are
// stored): rows blockIdx.x, blockIdx.x + grid, ... of the fp16 output are
// normalised by all threads of the CTA with fp32 statistics (biased
// variance, two passes over registers) and written to p.ln.y.
constexpr int kLnVec = 4;  // 16-byte vectors per thread: h <= 448 * 4 * 8
__device__ void ln_phase(const GemmParams& p, const Ctl& c) {
  __syncthreads();
  volatile int* ok_flag = c.last_flag;
  if (threadIdx.x == 0) {
    const bool mine = *c.abort_flag == 0;
    const bool met = grid_sync(p.ln.sync, gridDim.x, drain_ns(p.wait_ns));
    if (!met) set_error(p.err, DEV_TIMEOUT_EPILOGUE);
    *ok_flag = mine && met;
  }
  __syncthreads();
  if (!*ok_flag) return;
  float* red = c.stage;
  const int nvec = p.n / 8;
  for (int r = blockIdx.x; r < p.m; r += gridDim.x) {
    const uint4* xr = reinterpret_cast<const uint4*>(p.y + static_cast<size_t>(r) * p.ldy);
    float v[kLnVec][8];
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kLnVec; ++i) {
      const int vi = threadIdx.x + i * kThreads;
      if (vi < nvec) {
        const uint4 u = __ldcg(xr + vi);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(u32_as_h2(w[e]));
          v[i][2 * e] = f.x;
          v[i][2 * e + 1] = f.y;
          sum += f.x + f.y;
        }
      }
    }
    const float mean = block_sum_all(sum, red) / static_cast<float>(p.n);
    float sq = 0.f;
#pragma unroll
    for (int i = 0; i < kLnVec; ++i) {
      if (threadIdx.x + i * kThreads < nvec) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float dl = v[i][e] - mean;
          sq += dl * dl;
        }
      }
    }
    const float var = block_sum_all(sq, red + 32) / static_cast<float>(p.n);
    const float rstd = 1.0f / sqrtf(var + p.ln.eps);
    uint4* yr = reinterpret_cast<uint4*>(p.ln.y + static_cast<size_t>(r) * p.ln.ldy);
#pragma unroll
    for (int i = 0; i < kLnVec; ++i) {
      const int vi = threadIdx.x + i * kThreads;
      if (vi < nvec) {
        const uint4 gu = reinterpret_cast<const uint4*>(p.ln.g)[vi];
        const uint4 bu = reinterpret_cast<const uint4*>(p.ln.b)[vi];
        const uint32_t gw[4] = {gu.x, gu.y, gu.z, gu.w};
        const uint32_t bw[4] = {bu.x, bu.y, bu.z, bu.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 gf = __half22float2(u32_as_h2(gw[e]));
          const float2 bf = __half22float2(u32_as_h2(bw[e]));
          o[e] = h2_as_u32(__floats2half2_rn((v[i][2 * e] - mean) * rstd * gf.x + bf.x,
                                             (v[i][2 * e + 1] - mean) * rstd * gf.y + bf.y));
        }
        yr[vi] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

// Teardown: free TMEM once every thread is done (the
// MMA-issuing threads have waited for their own MMAs before getting here).
__device__ __forceinline__ void teardown(const GemmParams& p, const Ctl& c, uint32_t tmem_base, int warp) {
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_alloc);
  }
}

// ---------------------------------------------------------------------------
// the kernel: A tiles in shared memory, one MMA-issuing thread
// ---------------------------------------------------------------------------
// Walks a CTA's k-steps in order across its segments.
struct StepCursor {
  int q = 0, ks = 0;
  Seg g;
  bool valid = false;
  __device__ __forceinline__ void start(const Sched& sc, int cta) {
    q = 0;
    valid = get_seg(sc, cta, 0, g);
    ks = valid ? g.kb0 : 0;
  }
  __device__ __forceinline__ void next(const Sched& sc, int cta) {
    if (++ks < g.kb1) return;
    ++q;
    valid = get_seg(sc, cta, q, g);
    if (valid) ks = g.kb0;
  }
};

// KS: 64-wide k-blocks per k-step (two halve the mbarrier hand-offs per
// tile, which bound decode-sized tiles).  Three rings:
//   W  weight chunks in shared memory (4-bit: the packed codes + (min,
//      scale); fp16: TMA tiles that are the MMA's A operand directly), filled
//      by the producer far ahead of use: the weights stream from HBM, so the
//      bytes this SM keeps in flight set the rate at which it receives them;
//   B  activation boxes in shared memory (from L2, a short ring);
//   A  dequantized fp16 tiles (4-bit only), written by the dequantizing warps:
//      in shared memory, or with kTA in tensor memory (tcgen05.st, one weight
//      row per TMEM lane), read there by the MMA.  Decode-sized tiles use
//      kTA: the shared-memory port then carries only the copies, the code
//      reads and the MMA's B reads, not 2 x 16 KB of A per k-block.
// Each ring has its own issuing thread: B(i) waits for the MMA of step
// i - SB, W(i) for the dequantizing warps to have read step i - SW (they
// release a W slot as soon as its codes are in registers; with fp16 weights
// the MMA releases it), so the weight ring runs a whole ring ahead.
template <bool kW4, int KS, bool kTA>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                   const GemmParams p) {
  static_assert(!kTA || (kW4 && (KS == 2 || KS == 4)), "A in tensor memory: 4-bit weights, 2 or 4 k-blocks per step");
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int SW = p.w_stages, SB = p.b_stages, SA = p.a_stages;
  constexpr uint32_t a_slot_bytes = KS * kATileBytes;
  uint8_t* a_ring = smem;                                         // SA x KS fp16 A tiles (4-bit, !kTA)
  uint8_t* w_ring = a_ring + (kTA ? 0 : SA * a_slot_bytes);       // SW x w_slot_bytes
  uint8_t* b_ring = w_ring + SW * p.w_slot_bytes;        // SB x b_slot_bytes
  uint8_t* region = b_ring + SB * p.b_slot_bytes;
  uint64_t* wfull = reinterpret_cast<uint64_t*>(region);
  uint64_t* wempty = wfull + SW;
  uint64_t* bfull = wempty + SW;
  uint64_t* bempty = bfull + SB;
  uint64_t* afull = bempty + SB;
  uint64_t* aempty = afull + SA;
  uint64_t* drained = aempty + SA;
  const Ctl c = make_ctl(region, drained + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const uint32_t b_bytes = static_cast<uint32_t>(p.tok_tile) * 128u;  // one 64-wide activation box

  if (threadIdx.x == 0) {
    // barriers the MMA issuers commit to count one arrival per issuer
    for (int s = 0; s < SW; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], kW4 ? kDequantThreads : p.issuers);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(&bfull[s], 1);
      mbar_init(&bempty[s], p.issuers);
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(&afull[s], kDequantThreads);
      mbar_init(&aempty[s], p.issuers);
    }
    mbar_init(drained, p.issuers);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&c.accf[b], p.issuers);
      mbar_init(&c.acce[b], kEpiThreads);
    }
    *c.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(c.tmem_slot, p.tmem_alloc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *c.tmem_slot;
  const Sched& sc = p.sc;
  // The successor may launch now: its CTAs take SMs as this kernel's leave
  // and stream their weights while these finish.
  pdl_trigger();

  if (warp == 0 || warp == kBWarp) {
    // ------------------------------------------------------------ producers
    // Two issuing threads, one per ring: a thread completes about one copy
    // per HBM/L2 round trip whatever its size (up to ~16 KB), so the weight
    // stream and the activation stream each get their own, and every copy
    // moves a whole k-step (KS k-blocks: one bulk copy of the packed chunks,
    // one 3-D tensor box of the activations or fp16 weights).
    if (lane == 0) {
      const bool w_role = warp == 0;
      // weights are never written by kernels: only the activations wait for
      // the predecessor
      if (!w_role) pdl_wait();
      const uint64_t pol = w_role ? policy_evict_first() : policy_evict_last();
      if (w_role && !kW4) prefetch_tmap(&tmap_w);
      if (!w_role) prefetch_tmap(&tmap_x);
      const int S = w_role ? SW : SB;
      uint64_t* full = w_role ? wfull : bfull;
      uint64_t* empty = w_role ? wempty : bempty;
      uint8_t* ring = w_role ? w_ring : b_ring;
      const uint32_t slot_bytes = w_role ? p.w_slot_bytes : p.b_slot_bytes;
      const uint32_t tx = w_role ? KS * (kW4 ? static_cast<uint32_t>(kTileBytes) : static_cast<uint32_t>(kATileBytes))
                                 : KS * b_bytes;
      StepCursor cur;
      cur.start(sc, cta);
      Ring r;
      int n = 0;
      while (cur.valid) {
        if (!mbar_wait(&empty[r.s], r.ph ^ 1u, p.wait_ns)) {
          set_error(p.err, DEV_TIMEOUT_PRODUCER);
          *c.abort_flag = 1;
        }
        if (*c.abort_flag) break;
        uint8_t* dst = ring + r.s * slot_bytes;
        mbar_arrive_expect_tx(&full[r.s], tx);
        if (!w_role) {
          tma_load_3d(dst, &tmap_x, &full[r.s], 0, (cur.g.tile / sc.n_tiles) * p.tok_tile, cur.ks * KS, pol);
        } else if (kW4) {
          const int n_tile = cur.g.tile % sc.n_tiles;
          bulk_load(dst, p.wq + (static_cast<size_t>(n_tile) * p.kb_real + cur.ks * KS) * kTileBytes, KS * kTileBytes,
                    &full[r.s], pol);
        } else {
          tma_load_3d(dst, &tmap_w, &full[r.s], 0, (cur.g.tile % sc.n_tiles) * 128, cur.ks * KS, pol);
        }
        r.next(S);
        ++n;
        cur.next(sc, cta);
      }
      // Never leave the CTA with bulk copies still landing in its shared memory.
      for (int j = max(0, n - S); j < n; ++j)
        mbar_wait(&full[j % S], static_cast<uint32_t>(j / S) & 1u, drain_ns(p.wait_ns));
    }
  } else if (warp == 1 || warp == kMmaWarp2) {
    // ------------------------------------------------------------ MMA issuers
    // One issuing thread completes about one tcgen05.mma per ~120 cycles
    // whatever N, so decode tiles use two (warps 1 and 15): issuer mi takes
    // the k-blocks u of a step with u % issuers == mi into its own
    // accumulator (chain_cols apart); the epilogue adds the two.
    const int mi = warp == 1 ? 0 : 1;
    if (lane == 0 && mi < p.issuers) {
      const uint32_t idesc = idesc_f16_m128(static_cast<uint32_t>(p.tok_tile));
      // descriptors of slot 0; a slot is reached by adding its byte offset >> 4
      const uint64_t adesc0 = sw128_kmajor_desc(smem_u32(kW4 && !kTA ? a_ring : w_ring));
      const uint32_t a_tmem0 = tmem_base + p.a_col0;
      const uint64_t bdesc0 = sw128_kmajor_desc(smem_u32(b_ring));
      const uint32_t a_step = (kW4 ? a_slot_bytes : p.w_slot_bytes) >> 4;
      const uint32_t b_step = p.b_slot_bytes >> 4;
      const int SAx = kW4 ? SA : SW;  // the ring the A operand sits in
      Ring rb, ra;
      Seg g;
      bool stop = false;
      for (int q = 0; get_seg(sc, cta, q, g); ++q) {
        int buf;
        uint32_t par;
        acc_slot(q, p.acc_bufs, buf, par);
        if (!stop && !mbar_wait(&c.acce[buf], par ^ 1u, p.wait_ns)) {
          set_error(p.err, DEV_TIMEOUT_MMA);
          *c.abort_flag = 1;
        }
        if (*c.abort_flag) stop = true;
        tc_fence_after();
        const uint32_t d_tmem =
            tmem_base + static_cast<uint32_t>(buf) * p.acc_cols + static_cast<uint32_t>(mi) * p.chain_cols;
        for (int ks = g.kb0; ks < g.kb1 && !stop; ++ks, rb.next(SB), ra.next(SAx)) {
          bool ok = kW4 ? mbar_wait(&afull[ra.s], ra.ph, p.wait_ns) : mbar_wait(&wfull[ra.s], ra.ph, p.wait_ns);
          ok = ok && mbar_wait(&bfull[rb.s], rb.ph, p.wait_ns);
          if (!ok) {
            set_error(p.err, DEV_TIMEOUT_MMA);
            *c.abort_flag = 1;
          }
          if (*c.abort_flag) {
            stop = true;
            break;
          }
          const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(rb.s * b_step);
          if constexpr (kTA) {
            tc_fence_after();  // the dequantizing warps' tensor-memory stores
            const uint32_t a_tmem = a_tmem0 + static_cast<uint32_t>(ra.s * KS * 32);
#pragma unroll
            for (int u = 0; u < KS; ++u)
              if (u % p.issuers == mi) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_f16_ts(d_tmem, a_tmem + u * 32 + 8 * kk, bdesc + u * (b_bytes >> 4) + 2 * kk, idesc,
                             (ks > g.kb0 || u >= p.issuers || kk > 0) ? 1u : 0u);
              }
          } else {
            const uint64_t adesc = adesc0 + static_cast<uint64_t>(ra.s * a_step);
#pragma unroll
            for (int u = 0; u < KS; ++u)
              if (u % p.issuers == mi) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_f16_ss(d_tmem, adesc + u * (kATileBytes >> 4) + 2 * kk, bdesc + u * (b_bytes >> 4) + 2 * kk,
                             idesc, (ks > g.kb0 || u >= p.issuers || kk > 0) ? 1u : 0u);
              }
          }
          mma_commit(&bempty[rb.s]);
          mma_commit(kW4 ? &aempty[ra.s] : &wempty[ra.s]);
        }
        // Every segment ends with a commit, also after an abort, so the
        // epilogue never waits on a barrier nobody signals.
        mma_commit(&c.accf[buf]);
      }
      // all MMAs have completed before TMEM can be released
      mma_commit(drained);
      mbar_wait(drained, 0, drain_ns(p.wait_ns));
    }
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------------------------ dequantize
    if constexpr (kTA) {
      // warp w stores TMEM lanes 32 (w % 4) ..: one weight row per thread;
      // the two warps of a lane quarter take alternate k-blocks of the step
      constexpr int KU = KS / 2;  // k-blocks per thread and step
      const int quarter = warp & 3;
      const int grp = (warp - 2) >> 2;
      const int row = quarter * 32 + lane;
      const uint32_t t_row = tmem_base + p.a_col0 + (static_cast<uint32_t>(quarter * 32) << 16);
      Ring rw, ra;
      Seg g;
      bool stop = false;
      for (int q = 0; !stop && get_seg(sc, cta, q, g); ++q) {
        for (int ks = g.kb0; ks < g.kb1; ++ks, rw.next(SW), ra.next(SA)) {
          bool ok = mbar_wait(&wfull[rw.s], rw.ph, p.wait_ns);
          ok = ok && mbar_wait(&aempty[ra.s], ra.ph ^ 1u, p.wait_ns);
          if (!ok) {
            set_error(p.err, DEV_TIMEOUT_CONSUMER);
            *c.abort_flag = 1;
          }
          // warp-uniform: the tensor-memory store below is a warp-wide instruction
          if (__any_sync(0xffffffffu, !ok || *c.abort_flag)) {
            stop = true;
            break;
          }
          tc_fence_after();  // the MMAs that read this A slot have completed
          uint4 c0[KU], c1[KU];
          __half2 mm[KU];
#pragma unroll
          for (int v = 0; v < KU; ++v) {
            const uint8_t* raw = w_ring + rw.s * p.w_slot_bytes + (grp + 2 * v) * kTileBytes;
            c0[v] = *reinterpret_cast<const uint4*>(raw + row * 32);
            c1[v] = *reinterpret_cast<const uint4*>(raw + row * 32 + 16);
            mm[v] = *reinterpret_cast<const __half2*>(raw + kTileCodeBytes + row * 4);
          }
          // the codes are in registers: the weight slot may be refilled
          mbar_arrive(&wempty[rw.s]);
#pragma unroll
          for (int v = 0; v < KU; ++v) {
            const __half2 m2 = __low2half2(mm[v]);
            const __half2 s2 = __high2half2(mm[v]);
            const uint32_t words[8] = {c0[v].x, c0[v].y, c0[v].z, c0[v].w, c1[v].x, c1[v].y, c1[v].z, c1[v].w};
            uint32_t r[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const uint4 d = dequant8(words[j], s2, m2);
              r[4 * j] = d.x;
              r[4 * j + 1] = d.y;
              r[4 * j + 2] = d.z;
              r[4 * j + 3] = d.w;
            }
            __syncwarp();
            tmem_st_x32(t_row + static_cast<uint32_t>(ra.s * KS * 32 + (grp + 2 * v) * 32), r);
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&afull[ra.s]);
        }
      }
    } else if (kW4) {
      const int ct = threadIdx.x - 64;
      const int row = ct >> 1;
      const int hf = ct & 1;
      Ring rw, ra;
      Seg g;
      bool stop = false;
      for (int q = 0; !stop && get_seg(sc, cta, q, g); ++q) {
        for (int ks = g.kb0; ks < g.kb1; ++ks, rw.next(SW), ra.next(SA)) {
          bool ok = mbar_wait(&wfull[rw.s], rw.ph, p.wait_ns);
          ok = ok && mbar_wait(&aempty[ra.s], ra.ph ^ 1u, p.wait_ns);
          if (!ok) {
            set_error(p.err, DEV_TIMEOUT_CONSUMER);
            *c.abort_flag = 1;
          }
          if (*c.abort_flag) {
            stop = true;
            break;
          }
          const uint8_t* raw = w_ring + rw.s * p.w_slot_bytes;
          uint4 cw[KS];
          __half2 mm[KS];
#pragma unroll
          for (int u = 0; u < KS; ++u) {
            cw[u] = *reinterpret_cast<const uint4*>(raw + u * kTileBytes + row * 32 + hf * 16);
            mm[u] = *reinterpret_cast<const __half2*>(raw + u * kTileBytes + kTileCodeBytes + row * 4);
          }
          // the codes are in registers: the weight slot may be refilled
          mbar_arrive(&wempty[rw.s]);
#pragma unroll
          for (int u = 0; u < KS; ++u) {
            const __half2 m2 = __low2half2(mm[u]);
            const __half2 s2 = __high2half2(mm[u]);
            uint8_t* arow = a_ring + ra.s * a_slot_bytes + u * kATileBytes + row * 128;
            const uint32_t words[4] = {cw[u].x, cw[u].y, cw[u].z, cw[u].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int phys = (hf * 4 + j) ^ (row & 7);
              *reinterpret_cast<uint4*>(arow + phys * 16) = dequant8(words[j], s2, m2);
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(&afull[ra.s]);
        }
      }
    }
  } else if (warp < kEpiWarp0 + 4) {
    epilogue_role(p, c, tmem_base, warp, lane);
  }
  teardown(p, c, tmem_base, warp);
  if (p.ln_on) ln_phase(p, c);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// fp16 matrix [rows][cols] (row stride ld elements, cols a multiple of 64)
// viewed as [cols / 64][rows][64]: a box {64, box_rows, box_kb} is box_kb
// consecutive 64-column blocks, each a 128-byte-swizzled [box_rows][64] tile
// (the UMMA K-major layout), stacked in shared memory; zero fill out of bounds.
bool encode_tmap(CUtensorMap* map, const void* base, int rows, int cols, int ld, int box_rows, int box_kb) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(cols / 64)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 2, 128};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(box_kb)};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Encoded maps keyed by everything that goes into them, so repeated calls on
// the same buffers (every decode step) skip the encoding.  A map holds only
// the address, extents, stride and box, so a key always yields the same map.
struct TmapKey {
  const void* base;
  int rows, cols, ld, box_rows, box_kb;
  bool operator==(const TmapKey& o) const {
    return base == o.base && rows == o.rows && cols == o.cols && ld == o.ld && box_rows == o.box_rows &&
           box_kb == o.box_kb;
  }
};
constexpr int kTmapCache = 64;
struct TmapCache {
  std::mutex mu;
  TmapKey key[kTmapCache];
  CUtensorMap map[kTmapCache];
  bool used[kTmapCache] = {};
  int next = 0;
};
TmapCache g_tmaps;

bool make_tmap(CUtensorMap* map, const void* base, int rows, int cols, int ld, int box_rows, int box_kb) {
  const TmapKey k{base, rows, cols, ld, box_rows, box_kb};
  std::lock_guard<std::mutex> lock(g_tmaps.mu);
  for (int i = 0; i < kTmapCache; ++i) {
    if (g_tmaps.used[i] && g_tmaps.key[i] == k) {
      *map = g_tmaps.map[i];
      return true;
    }
  }
  if (!encode_tmap(map, base, rows, cols, ld, box_rows, box_kb)) return false;
  const int i = g_tmaps.next;
  g_tmaps.next = (i + 1) % kTmapCache;
  g_tmaps.key[i] = k;
  g_tmaps.map[i] = *map;
  g_tmaps.used[i] = true;
  return true;
}

struct Plan {
  int tok_tile, tok_tiles, n_tiles;
  int ks;       // k-blocks per stage of gemm_tc_kernel
  bool tmem_a;  // dequantized A in tensor memory
  Sched sc;
  int w_stages, b_stages, a_stages;
  uint32_t w_slot_bytes, b_slot_bytes;
  uint32_t acc_cols, chain_cols, tmem_alloc, a_col0;
  int issuers, acc_bufs;
  size_t smem;
  size_t partial_bytes, counter_bytes;
};

int round_up(int a, int b) { return (a + b - 1) / b * b; }
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

Plan make_plan(int m, int n, int k, int w_bits, int force_splits, int force_tok_tile) {
  Plan P{};
  const int kb_real = k / 64;
  if (force_tok_tile > 0) {
    P.tok_tile = force_tok_tile;
    P.tok_tiles = (m + P.tok_tile - 1) / P.tok_tile;
  } else if (m <= 256) {
    P.tok_tile = round_up(max(m, 16), 16);
    P.tok_tiles = 1;
  } else {
    P.tok_tiles = (m + 255) / 256;
    P.tok_tile = round_up((m + P.tok_tiles - 1) / P.tok_tiles, 16);
  }
  // Decode-sized tiles move several k-blocks per copy (a copying thread
  // completes about one copy per round trip, so bytes per copy set the rate):
  // 4-bit weights four where the dequantized A ring still fits tensor memory
  // with four k-blocks per slot (tokens <= 128), else two; fp16 weights two.
  const bool dec = P.tok_tile <= kDecodeMaxTok;
  if (dec && w_bits == 4 && P.tok_tile <= 128 && kb_real % 4 == 0) P.ks = 4;
  else if (dec && kb_real % 2 == 0) P.ks = 2;
  else P.ks = 1;
  const int kb_total = kb_real / P.ks;  // k-steps per tile
  const int min_iters = max(1, kMinItersPerCta / P.ks);
  P.n_tiles = (n + 127) / 128;
  const int tiles = P.n_tiles * P.tok_tiles;
  const int sms = runtime().num_sms;
  Sched& s = P.sc;
  s.tiles = tiles;
  s.n_tiles = P.n_tiles;
  s.kb_total = kb_total;
  s.iters = static_cast<long long>(tiles) * kb_total;
  s.splits = 1;
  s.per = kb_total;
  const size_t tile_bytes = static_cast<size_t>(P.tok_tile) * 128 * sizeof(float);
  if (force_splits > 1) {
    s.mode = SCHED_SPLITS;
    s.per = (kb_total + force_splits - 1) / force_splits;
    s.splits = min(kMaxContrib, (kb_total + s.per - 1) / s.per);
    s.per = (kb_total + s.splits - 1) / s.splits;
    s.grid = tiles * s.splits;
    if (s.splits > 1) P.partial_bytes = static_cast<size_t>(s.grid) * tile_bytes;
    else s.mode = SCHED_TILES, s.grid = min(tiles, sms);
  } else if (force_splits == 1 || tiles >= 16 * sms ||
             tiles % std::max<long long>(1, std::min<long long>(sms, s.iters / min_iters)) == 0) {
    // many tiles, or whole tiles already divide evenly over the CTAs stream-K would use
    s.mode = SCHED_TILES;
    s.grid = min(tiles, sms);
  } else {
    s.mode = SCHED_STREAMK;
    s.grid = static_cast<int>(std::min<long long>(sms, std::max<long long>(1, s.iters / min_iters)));
    // A tile is shared by at most ceil(kb_total / (iters / grid)) + 1 CTAs.
    const long long per_cta = s.iters / s.grid;
    if ((kb_total + per_cta - 1) / per_cta + 1 > kMaxContrib)
      s.grid = static_cast<int>(std::max<long long>(1, s.iters * (kMaxContrib - 2) / kb_total));
    // Few tiles (at most half as many as SMs): exactly two CTAs per tile (each
    // half its k-steps) may finish sooner than spreading over every SM, since
    // a tile with c contributors ends with the finalizer reading the others'
    // partials, one L2 round trip (~1.5 k-steps, measured) per 16-token chunk
    // and pair of contributors, while two contributors take the prefetched
    // path.  Estimated in k-steps.
    if (2 * tiles <= s.grid && kb_total % 2 == 0) {
      const double per_all = static_cast<double>(s.iters) / s.grid;
      const int contrib_all = static_cast<int>((kb_total + per_all - 1) / per_all) + 1;
      const double chunks = P.tok_tile / 16.0;
      const double cost_all = per_all + ((contrib_all - 1 + 1) / 2) * chunks * 1.5;
      const double cost_two = kb_total / 2.0 + 0.2 * chunks;
      if (cost_two < cost_all) s.grid = 2 * tiles;
    }
    P.partial_bytes = static_cast<size_t>(2) * s.grid * tile_bytes;
  }
  if (P.partial_bytes > 0) P.counter_bytes = static_cast<size_t>(tiles) * 2 * sizeof(int);
  // Shared memory: the A ring (4-bit), a short activation ring, and as deep a
  // weight ring as the rest allows (the bytes of weights in flight per SM set
  // the rate at which they arrive from HBM).  Three activation slots when
  // that still leaves room for at least 8 weight k-steps, else two.
  const int budget = kMaxSmem - 1024 - kBarrierBytes - kEpiStageBytes;
  // Decode-sized 4-bit tiles keep the dequantized A in tensor memory after
  // the two accumulator buffers (512 columns: 2 x round_up(tokens, 32) + A
  // slots of 64 columns); larger tiles need the columns for accumulators.
  // Tensor memory (512 columns) for 4-bit decode tiles: the two issuers'
  // accumulators per buffer, two buffers where they fit with two A slots
  // (tokens <= 64), else one, then the A ring.
  P.tmem_a = dec && w_bits == 4 && P.ks >= 2;
  if (P.tmem_a) {
    P.chain_cols = static_cast<uint32_t>(round_up(P.tok_tile, 32));
    P.issuers = 2;
    P.acc_cols = static_cast<uint32_t>(P.issuers) * P.chain_cols;
    P.acc_bufs = 2 * P.acc_cols + 2u * 32u * P.ks <= 512u ? 2 : 1;
    P.a_col0 = static_cast<uint32_t>(P.acc_bufs) * P.acc_cols;
    P.tmem_alloc = 512;
  } else {
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(P.tok_tile)) cols <<= 1;
    P.issuers = 1;
    P.chain_cols = cols;
    P.acc_cols = cols;
    P.acc_bufs = 2;
    P.tmem_alloc = 2 * cols;
  }
  const int a_slot = w_bits == 4 && !P.tmem_a ? P.ks * kATileBytes : 0;
  P.a_stages = w_bits != 4 ? 0 : P.tmem_a ? std::min(4, static_cast<int>((512 - P.a_col0) / (32 * P.ks))) : 3;
  P.w_slot_bytes = static_cast<uint32_t>(w_bits == 4 ? round_up(P.ks * kTileBytes, 1024) : P.ks * kATileBytes);
  P.b_slot_bytes = static_cast<uint32_t>(P.ks * P.tok_tile * 128);
  const int rest = budget - P.a_stages * a_slot;
  const int w_slot = static_cast<int>(P.w_slot_bytes), b_slot = static_cast<int>(P.b_slot_bytes);
  P.b_stages = rest - 3 * b_slot >= 4 * w_slot ? 3 : 2;
  P.w_stages = min(kMaxWStages, (rest - P.b_stages * b_slot) / w_slot);
  P.smem = static_cast<size_t>(P.a_stages) * a_slot + static_cast<size_t>(P.w_stages) * w_slot +
           static_cast<size_t>(P.b_stages) * b_slot + 1024 + kBarrierBytes + kEpiStageBytes;
  return P;
}

// Raises the kernel's dynamic shared-memory limit once per process; one
// instantiation (and so one flag) per kernel.
template <auto kKernel>
cudaError_t configure_once() {
  static cudaError_t status = cudaErrorNotReady;
  static std::once_flag once;
  std::call_once(once, [] {
    status = cudaFuncSetAttribute(kKernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  });
  return status;
}

// A fused LayerNorm needs every CTA resident at once (grid barrier), so that
// variant is a cooperative launch; the grid never exceeds one CTA per SM.
template <bool kW4, int KS, bool kTA>
cudaError_t launch_general(const Plan& P, const CUtensorMap& tx, const CUtensorMap& tw, const GemmParams& p,
                           cudaStream_t s) {
  const cudaError_t e = configure_once<gemm_tc_kernel<kW4, KS, kTA>>();
  if (e != cudaSuccess) return e;
  if (!p.ln_on) return launch_pdl(gemm_tc_kernel<kW4, KS, kTA>, dim3(P.sc.grid), dim3(kThreads), P.smem, s, tx, tw, p);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.sc.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = P.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t le = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<kW4, KS, kTA>, tx, tw, p);
  if (le != cudaSuccess) return le;
  return launched();
}

}  // namespace

size_t linear_workspace_bytes(int m, int n, int k, int w_bits, int force_splits) {
  const Plan P = make_plan(m, n, k, w_bits, force_splits, 0);
  if (P.partial_bytes == 0) return 0;
  return align256(P.partial_bytes) + align256(P.counter_bytes);
}

size_t linear_counter_bytes(int m, int n, int k, int w_bits, int force_splits) {
  return make_plan(m, n, k, w_bits, force_splits, 0).counter_bytes;
}

size_t linear_partial_bytes(int m, int n, int k, int w_bits, int force_splits) {
  return make_plan(m, n, k, w_bits, force_splits, 0).partial_bytes;
}

cudaError_t launch_linear(const LinearArgs& a, void* ws, size_t ws_bytes, cudaStream_t s) {
  if (a.m == 0 || a.n == 0) return cudaSuccess;
  const Plan P = make_plan(a.m, a.n, a.k, a.w_bits, a.force_splits, a.force_tok_tile);
  const bool w4 = a.w_bits == 4;
  if (P.w_stages < 2 || P.b_stages < 2) return cudaErrorInvalidValue;
  // mbarriers the kernel lays out before its control words (make_ctl):
  // full/empty per weight and activation slot, afull/aempty per A slot, the drain barrier,
  // accf/acce x 2
  const int n_bars = 2 * (P.w_stages + P.b_stages + P.a_stages) + 5;
  if (n_bars > kMaxBarriers) return cudaErrorInvalidValue;
  CUtensorMap tx, tw;
  if (!make_tmap(&tx, a.x, a.m, a.k, a.ldx, P.tok_tile, P.ks)) return cudaErrorInvalidValue;
  if (w4) {
    tw = tx;
  } else if (!make_tmap(&tw, a.w, a.n, a.k, a.k, 128, P.ks)) {
    return cudaErrorInvalidValue;
  }
  GemmParams p{};
  p.wq = static_cast<const uint8_t*>(a.w);
  p.m = a.m;
  p.n = a.n;
  p.k = a.k;
  p.tok_tile = P.tok_tile;
  p.kb_real = a.k / 64;
  p.w_stages = P.w_stages;
  p.b_stages = P.b_stages;
  p.a_stages = P.a_stages;
  p.w_slot_bytes = P.w_slot_bytes;
  p.b_slot_bytes = P.b_slot_bytes;
  p.acc_cols = P.acc_cols;
  p.chain_cols = P.chain_cols;
  p.issuers = P.issuers;
  p.acc_bufs = P.acc_bufs;
  p.tmem_alloc = P.tmem_alloc;
  p.a_col0 = P.a_col0;
  p.sc = P.sc;
  p.bias = a.bias;
  p.residual = a.residual;
  p.ld_res = a.ld_res;
  p.epi = a.epi;
  p.wait_ns = runtime().wait_limit_ns;
  p.err = runtime().err;
  if (a.epi & EPI_F32_OUT) {
    p.yf = static_cast<float*>(a.y);
    p.ldyf = a.ldy;
  } else {
    p.y = static_cast<__half*>(a.y);
    p.ldy = a.ldy;
  }
  if (P.partial_bytes > 0) {
    if (a.counters != nullptr) {
      if (ws == nullptr || ws_bytes < P.partial_bytes) return cudaErrorInvalidValue;
      p.partials = static_cast<float*>(ws);
      p.counters = a.counters;
    } else {
      const size_t need = align256(P.partial_bytes) + align256(P.counter_bytes);
      if (ws == nullptr || ws_bytes < need) return cudaErrorInvalidValue;
      p.partials = static_cast<float*>(ws);
      p.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + align256(P.partial_bytes));
      const cudaError_t e = cudaMemsetAsync(p.counters, 0, P.counter_bytes, s);
      if (e != cudaSuccess) return e;
    }
  }
  if (a.kv != nullptr) {
    // whole 64-feature groups of one head per K/V tile; one token tile
    if (a.m > kFuseMaxRows || P.tok_tiles != 1 || a.n != 3 * a.kv->h || a.kv->h % 128 != 0 ||
        (a.epi & ~EPI_BIAS) != 0)
      return cudaErrorInvalidValue;
    p.kv_on = 1;
    p.kv = *a.kv;
  }
  if (a.ln != nullptr) {
    if (a.m > kFuseMaxRows || (a.epi & EPI_F32_OUT) || a.n % 8 != 0 || a.n > kThreads * 8 * 4 ||
        a.ln->sync == nullptr || P.sc.grid > runtime().num_sms)
      return cudaErrorInvalidValue;
    p.ln_on = 1;
    p.ln = *a.ln;
  }
  if (w4 && P.tmem_a) {
    if (P.ks == 4) return launch_general<true, 4, true>(P, tx, tw, p, s);
    return launch_general<true, 2, true>(P, tx, tw, p, s);
  }
  if (w4) return launch_general<true, 1, false>(P, tx, tw, p, s);
  if (P.ks == 2) return launch_general<false, 2, false>(P, tx, tw, p, s);
  return launch_general<false, 1, false>(P, tx, tw, p, s);
}

}  // namespace flexq

// Top-k sparse decode attention over the 4-bit KV cache ("FlexGen研究学术报告"
// section 三(C): only the top 10 % of the cache by attention value is loaded,
// a Top-k sparse approximation).  For each (sequence, head):
//   s_t = q . k_hat_t / sqrt(d) for all L cached keys (K is read in full),
//   p_t = exp(s_t - max s) / sum_t exp(s_t - max s)   (softmax over all keys),
//   T   = the kk keys with the largest s_t (the lower index wins a tie),
//   o   = sum_{t in T} p_t v_hat_t                     (V read only for T).
// The kept weights are the full-softmax weights, not renormalised over T;
// with kk = L the result is dense attention.
//
// One CTA of 128 threads per (head, sequence).  Scores as in the dense
// kernel (q as 15-bit fixed point, dp4a over the nibbles, scale*dot +
// min*sum q per group), kept in shared memory.  Selection: 1024 equal-width
// value bins over [min, max] of the scores (a monotone map, so the kk-th
// largest score falls in the bin where the count from the top reaches kk);
// every key above that bin is kept, and the keys inside it are ranked exactly
// (order-preserving 32-bit key, the lower index first among equal keys).  V is token-
// interleaved in blocks of 8 tokens, so a block is read only when it holds a
// kept token; its weights are 16-bit fixed point normalised by the largest
// kept p * scale of each group, 0 for the tokens not kept.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "quant_common.cuh"

namespace flexq {
namespace {

constexpr int kTkThreads = 128;
constexpr int kBins = 1024;  // kBins / kTkThreads bins per thread in the bucket search
constexpr int kTkWarps = kTkThreads / 32;

__device__ __forceinline__ uint32_t order_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  __syncthreads();
  if (lane_id() == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
#pragma unroll
  for (int w = 0; w < kTkWarps; ++w) r += red[w];
  return r;
}

__device__ __forceinline__ float block_min(float v, float* red) {
  v = -warp_max(-v);
  __syncthreads();
  if (lane_id() == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kTkWarps; ++w) r = fminf(r, red[w]);
  return r;
}

__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  __syncthreads();
  if (lane_id() == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kTkWarps; ++w) r = fmaxf(r, red[w]);
  return r;
}

// Exclusive prefix sum over the CTA's threads in thread order; returns this
// thread's prefix, and the total through *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* scan, int* total) {
  const int lane = lane_id(), w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  __syncthreads();
  if (lane == 31) scan[w] = incl;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int k = 0; k < kTkWarps; ++k) {
    if (k < w) before += scan[k];
    all += scan[k];
  }
  *total = all;
  return before + incl - v;
}

template <int D>
__global__ void __launch_bounds__(kTkThreads) attn_topk_q4_kernel(const __half* __restrict__ q, int ldq, KvView kv,
                                                                  int heads, int len, int kk,
                                                                  __half* __restrict__ out, int ldo,
                                                                  int32_t* __restrict__ idx_out,
                                                                  float inv_sqrt_d, AppendRow app) {
  pdl_wait();  // q, the cache and the outputs follow the stream's earlier kernels
  constexpr int G = D / 64;
  constexpr int DPL = D / 4;
  constexpr int NW = DPL / 8;
  constexpr int DPV = D / 32;
  extern __shared__ float sc[];                                  // [len] scores
  int* blist = reinterpret_cast<int*>(sc + ((len + 3) & ~3));     // [nblk] blocks holding a kept key
  int* cand = blist + (((len + 7) / 8 + 3) & ~3);                   // [len] keys in the threshold bin
  uint8_t* sel = reinterpret_cast<uint8_t*>(cand + ((len + 3) & ~3));  // [len] kept flags
  __shared__ int hist[kBins];
  __shared__ int ncand;
  __shared__ int scan[kTkWarps];
  __shared__ float red[kTkWarps];
  __shared__ float stat[2 * G + 1];
  __shared__ uint32_t pick[3];  // bucket, keys above it, keys still needed
  __shared__ float partv[kTkWarps][D];
  const int j = blockIdx.x, i = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t hr = static_cast<size_t>(i) * heads + j;
  const uint32_t* kw = reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(kv.k) + hr * kv.max_len * (D / 2));
  const __half2* km = static_cast<const __half2*>(kv.k_meta) + hr * kv.max_len * G;
  const __half2* vm = static_cast<const __half2*>(kv.v_meta) + hr * kv.max_len * G;
  const uint32_t* vw = static_cast<const uint32_t*>(kv.v) + hr * (kv_pad_len(kv.max_len) / 8) * D;

  // decode: this token's K/V rows enter the cache before the scores read it
  if (app.pos >= 0) {
    append_group_q4<D>(app, kv, i, j, heads, warp, lane);
    __syncthreads();
  }

  // ---- scores (all keys)
  const int cq = lane & 3, g = (cq * DPL) / 64;
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
  const float qscale = ldexpf(1.0f, 14 - qexp), inv_qscale = ldexpf(1.0f, qexp - 14);
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
  // kUnroll groups of tokens are loaded before any is used, so each lane keeps
  // several loads in flight (the pass is bound by load latency otherwise)
  float mx = -INFINITY, mn = INFINITY;
  constexpr int kStride = kTkThreads / 4;  // tokens per block-wide step
  constexpr int kUnroll = 4;
  for (int base = warp * 8; base < len; base += kUnroll * kStride) {
    uint32_t cw[kUnroll][NW];
    __half2 msh[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = base + u * kStride + (lane >> 2);
      if (t < len) {
        const uint32_t* src = kw + static_cast<size_t>(t) * (D / 8) + cq * NW;
        if constexpr (NW == 4) {
          const uint4 v = *reinterpret_cast<const uint4*>(src);
          cw[u][0] = v.x; cw[u][1] = v.y; cw[u][2] = v.z; cw[u][3] = v.w;
        } else {
          const uint2 v = *reinterpret_cast<const uint2*>(src);
          cw[u][0] = v.x; cw[u][1] = v.y;
        }
        msh[u] = km[static_cast<size_t>(t) * G + g];
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
          const uint32_t lo = cw[u][w] & 0x0F0F0F0Fu, hi = (cw[u][w] >> 4) & 0x0F0F0F0Fu;
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
        if (cq == 0) sc[t] = s;
        mx = fmaxf(mx, s);
        mn = fminf(mn, s);
      }
    }
  }
  const float M = block_max(mx, red);  // its barriers also publish sc[]

  const float m0 = block_min(mn, red);

  // ---- selection.  bin(t) = min(kBins-1, floor((s_t - m0) * kBins / (M - m0)))
  // is non-decreasing in s_t (every step rounds monotonically), so the kk-th
  // largest score lies in bin B with (keys in bins > B) < kk <= (keys in
  // bins >= B); all scores equal puts every key in bin 0.
  const float bscale = M > m0 ? static_cast<float>(kBins) / (M - m0) : 0.f;
  auto bin_of = [&](float v) { return min(kBins - 1, static_cast<int>((v - m0) * bscale)); };
  for (int b = threadIdx.x; b < kBins; b += kTkThreads) hist[b] = 0;
  if (threadIdx.x == 0) ncand = 0;
  __syncthreads();
  for (int t0 = 0; t0 < len; t0 += kTkThreads) {
    const int t = t0 + threadIdx.x;
    const bool act = t < len;
    const int bin = act ? bin_of(sc[t]) : kBins + lane;
    // lanes that hit the same bin add once, by their lowest lane
    const unsigned same = __match_any_sync(0xffffffffu, bin);
    if (act && __ffs(same) - 1 == lane) atomicAdd(&hist[bin], __popc(same));
  }
  __syncthreads();
  {
    // thread i owns bins [kPer * i, kPer * i + kPer); a suffix sum over the
    // threads (the block scan on reversed thread order) finds the owner of B
    constexpr int kPer = kBins / kTkThreads;
    const int owner = kTkThreads - 1 - threadIdx.x;  // scan order: the top bins first
    int cnt[kPer], own = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      cnt[k] = hist[owner * kPer + k];
      own += cnt[k];
    }
    int total = 0;
    const int above = block_exclusive_scan(own, scan, &total);  // keys in the bins above this thread's
    if (above < kk && kk <= above + own) {
      int a = above, b = owner * kPer + kPer - 1;
      for (int k = kPer - 1; k > 0; --k, --b) {
        if (a + cnt[k] >= kk) break;
        a += cnt[k];
      }
      pick[0] = static_cast<uint32_t>(b);
      pick[1] = static_cast<uint32_t>(a);
    }
  }
  __syncthreads();
  const int B = static_cast<int>(pick[0]);
  const int need = kk - static_cast<int>(pick[1]);  // keys of bin B to keep
  for (int t = threadIdx.x; t < len; t += kTkThreads) {
    const int bin = bin_of(sc[t]);
    sel[t] = bin > B;
    if (bin == B) cand[atomicAdd(&ncand, 1)] = t;
  }
  __syncthreads();
  // exact rank inside bin B: keys above this one, then equal keys at a lower slot
  const int nc = ncand;
  for (int ci = threadIdx.x; ci < nc; ci += kTkThreads) {
    const int t = cand[ci];
    const uint32_t key = order_key(sc[t]);
    int r = 0;
    for (int cj = 0; cj < nc; ++cj) {
      const int u = cand[cj];
      const uint32_t ku = order_key(sc[u]);
      r += ku > key || (ku == key && u < t);
    }
    sel[t] = r < need;
  }
  // contiguous segments for the ordered index output
  const int seg = (len + kTkThreads - 1) / kTkThreads;
  const int t0 = threadIdx.x * seg, t1 = min(len, t0 + seg);

  // ---- softmax sum over all keys; per group sum p*min and max p*scale over the kept keys
  float s_all = 0.f;
  float pm[G], wm[G];
#pragma unroll
  for (int gg = 0; gg < G; ++gg) pm[gg] = wm[gg] = 0.f;
  __syncthreads();  // sel[] complete
  for (int t = threadIdx.x; t < len; t += kTkThreads) {
    const float p = __expf(sc[t] - M);
    s_all += p;
    if (sel[t]) {
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        const float2 ms = __half22float2(vm[static_cast<size_t>(t) * G + gg]);
        pm[gg] += p * ms.x;
        wm[gg] = fmaxf(wm[gg], p * ms.y);
      }
    }
  }
  const float S = block_sum(s_all, red);
#pragma unroll
  for (int gg = 0; gg < G; ++gg) {
    const float a = block_sum(pm[gg], red);
    const float b = block_max(wm[gg], red);
    if (threadIdx.x == 0) {
      stat[gg] = a;
      stat[G + gg] = b;
    }
  }
  __syncthreads();

  // ---- kept indices in ascending order
  if (idx_out != nullptr) {
    int n_sel = 0;
    for (int t = t0; t < t1; ++t) n_sel += sel[t];
    int all = 0;
    int at = block_exclusive_scan(n_sel, scan, &all);
    int32_t* dst = idx_out + hr * kk;
    for (int t = t0; t < t1; ++t)
      if (sel[t]) dst[at++] = t;
  }

  // ---- the 8-token blocks holding a kept token, in ascending order
  const int nblk = (len + 7) / 8;
  int n_kb = 0;
  for (int b0 = 0; b0 < nblk; b0 += kTkThreads) {
    const int blk = b0 + threadIdx.x;
    int any = 0;
    if (blk < nblk)
      for (int k = 0; k < 8 && blk * 8 + k < len; ++k) any |= sel[blk * 8 + k];
    int cnt = 0;
    const int at = block_exclusive_scan(any, scan, &cnt);
    if (any) blist[n_kb + at] = blk;
    n_kb += cnt;
  }
  __syncthreads();

  // ---- values of those blocks; kVU blocks' words in flight per lane
  constexpr int kVU = 4;
  const int gv = (lane * DPV) / 64;
  uint32_t al[DPV], ah[DPV];
#pragma unroll
  for (int e = 0; e < DPV; ++e) al[e] = ah[e] = 0u;
  for (int r0 = warp; r0 < n_kb; r0 += kVU * kTkWarps) {
    uint32_t words[kVU][DPV];
    int blks[kVU];
#pragma unroll
    for (int u = 0; u < kVU; ++u) {
      const int r = r0 + u * kTkWarps;
      blks[u] = r < n_kb ? blist[r] : -1;
      if (blks[u] >= 0) {
        const uint32_t* src = vw + static_cast<size_t>(blks[u]) * D + lane * DPV;
#pragma unroll
        for (int e = 0; e < DPV; ++e) words[u][e] = src[e];
      }
    }
#pragma unroll
    for (int u = 0; u < kVU; ++u) {
      if (blks[u] < 0) break;  // warp-uniform
      // lane k < 8 * G: token 8 blk + (k & 7), group k >> 3
      const int tk = blks[u] * 8 + (lane & 7);
      const int gk = lane >> 3;
      const bool kept = lane < 8 * G && tk < len && sel[tk];
      uint32_t wi = 0u;
      if (kept) {
        const float p = __expf(sc[tk] - M);
        const float sv = __high2float(vm[static_cast<size_t>(tk) * G + gk]);
        const float wqk = stat[G + gk] > 0.f ? 65535.0f / stat[G + gk] : 0.f;
        wi = min(65535u, __float2uint_rn(p * sv * wqk));
      }
      uint32_t le = 0u, lo = 0u, he = 0u, ho = 0u;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t w = __shfl_sync(0xffffffffu, wi, gv * 8 + k);
        const int sh = 8 * (k >> 1);
        if (k & 1) {
          lo |= (w & 0xFFu) << sh;
          ho |= (w >> 8) << sh;
        } else {
          le |= (w & 0xFFu) << sh;
          he |= (w >> 8) << sh;
        }
      }
#pragma unroll
      for (int e = 0; e < DPV; ++e) {
        const uint32_t lo4 = words[u][e] & 0x0F0F0F0Fu, hi4 = (words[u][e] >> 4) & 0x0F0F0F0Fu;
        al[e] = __dp4a(lo4, le, al[e]);
        al[e] = __dp4a(hi4, lo, al[e]);
        ah[e] = __dp4a(lo4, he, ah[e]);
        ah[e] = __dp4a(hi4, ho, ah[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < DPV; ++e)
    partv[warp][lane * DPV + e] = static_cast<float>(ah[e]) * 256.0f + static_cast<float>(al[e]);
  __syncthreads();
  for (int e = threadIdx.x; e < D; e += kTkThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kTkWarps; ++w) v += partv[w][e];
    const int gg = e / 64;
    const float o = v * (stat[G + gg] / 65535.0f) + stat[gg];
    out[static_cast<size_t>(i) * ldo + j * D + e] = __float2half_rn(o / S);
  }
}

template <int D>
cudaError_t launch_topk(const __half* q, int ldq, const KvView& kv, int b, int heads, int len, int kk, __half* out,
                        int ldo, int32_t* idx, const AppendRow& app, cudaStream_t s) {
  const size_t smem = static_cast<size_t>((len + 3) & ~3) * sizeof(float) +
                      static_cast<size_t>(((len + 7) / 8 + 3) & ~3) * sizeof(int) +
                      static_cast<size_t>((len + 3) & ~3) * sizeof(int) + static_cast<size_t>((len + 15) & ~15);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(attn_topk_q4_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(heads, b);
  return launch_pdl(attn_topk_q4_kernel<D>, grid, dim3(kTkThreads), smem, s, q, ldq, kv, heads, len, kk, out, ldo,
                    idx, 1.0f / sqrtf(static_cast<float>(D)), app);
}

}  // namespace

cudaError_t launch_attn_topk(const __half* q, int ldq, const KvView& kv, int b, int heads, int d, int len, int kk,
                             __half* out, int ldo, int32_t* idx, const AppendRow& app, cudaStream_t s) {
  if (b == 0) return cudaSuccess;
  return d == 128 ? launch_topk<128>(q, ldq, kv, b, heads, len, kk, out, ldo, idx, app, s)
                  : launch_topk<64>(q, ldq, kv, b, heads, len, kk, out, ldo, idx, app, s);
}

}  // namespace flexq

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
// Design (one CTA = 128 output features x up to 256 tokens; the weight is the
// MMA's A operand so that small decode batches become the MMA's N):
//   warp 0      TMA producer: one cp.async.bulk of the packed 4-bit tile
//               (codes + min/scale, 4608 contiguous bytes) and one tiled
//               cp.async.bulk.tensor of the fp16 activations per 64-wide
//               k-block, completion counted on an mbarrier;
//   warps 2-9   dequantize: (code | 0x6400) is the fp16 value 1024 + code, one
//               half2 subtract and one half2 fused multiply-add give
//               code * scale + min rounded once to fp16, written straight into
//               the 128-byte-swizzled K-major layout the tensor core reads;
//   warp 1      allocates TMEM and, from one thread, issues
//               tcgen05.mma.kind::f16 (M=128, N=tokens, K=16) x 4 per k-block,
//               freeing each stage with tcgen05.commit;
//   warps 2-9   epilogue: tcgen05.ld of the fp32 accumulator, + bias, GELU,
//               + residual, fp16 store (or fp32 atomic partial sums when K is
//               split across CTAs to fill the 148 SMs).
// Every mbarrier wait is bounded; on expiry the CTA records an error code in
// the device error word and unwinds (no trap).
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace flexq {
namespace {

constexpr int kThreads = 320;
constexpr int kConsumers = 256;
constexpr int kATileBytes = 128 * 64 * 2;
constexpr int kRawBytes = 5120;  // kTileBytes rounded up to keep 1 KB alignment
constexpr int kMaxSmem = 227 * 1024;
constexpr int kBarrierBytes = 256;

struct GemmParams {
  const uint8_t* wq;
  int m, n, k;
  int kb_total, kb_per_split;
  int tok_tile;
  int stages;
  uint32_t stage_bytes;
  uint32_t tmem_cols;
  const __half* bias;
  const __half* residual;
  int ld_res;
  __half* y;
  int ldy;
  float* yf;
  int ldyf;
  int epi;
  int splitk;
  uint64_t wait_ns;
  uint32_t* err;
};

__device__ __forceinline__ uint64_t drain_ns(uint64_t wait_ns) {
  return wait_ns > 1000000000ull ? wait_ns : 1000000000ull;
}

__device__ __forceinline__ float gelu_erf(float v) {
  return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}

__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) {
  return *reinterpret_cast<__half2*>(&u);
}
__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}

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

template <bool kW4>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                   const GemmParams p) {
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * p.stage_bytes);
  uint64_t* afull = full + S;
  uint64_t* empty = afull + S;
  uint64_t* accum = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x;
  const int t_tile = blockIdx.y;
  const int kb0 = blockIdx.z * p.kb_per_split;
  const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
  const int nkb = kb1 - kb0;
  const uint32_t b_bytes = static_cast<uint32_t>(p.tok_tile) * 128u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], kConsumers);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmap_x);
      if (!kW4) prefetch_tmap(&tmap_w);
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int issued = 0;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % S;
        const uint32_t r = static_cast<uint32_t>(i / S);
        if (!mbar_wait(&empty[s], (r & 1u) ^ 1u, p.wait_ns)) {
          set_error(p.err, DEV_TIMEOUT_PRODUCER);
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        uint8_t* st = smem + s * p.stage_bytes;
        const int kb = kb0 + i;
        if (kW4) {
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(kTileBytes) + b_bytes);
          bulk_load(st + kATileBytes + b_bytes,
                    p.wq + (static_cast<size_t>(n_tile) * p.kb_total + kb) * kTileBytes, kTileBytes,
                    &full[s], pol_w);
        } else {
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(kATileBytes) + b_bytes);
          tma_load_2d(st, &tmap_w, &full[s], kb * 64, n_tile * 128, pol_w);
        }
        tma_load_2d(st + kATileBytes, &tmap_x, &full[s], kb * 64, t_tile * p.tok_tile, pol_x);
        ++issued;
      }
      // Never leave the CTA with bulk copies still landing in its shared memory
      // (the drain keeps a deadline of its own so a short wait limit cannot cut
      // it short).
      for (int j = max(0, issued - S); j < issued; ++j)
        mbar_wait(&full[j % S], static_cast<uint32_t>(j / S) & 1u, drain_ns(p.wait_ns));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_m128(static_cast<uint32_t>(p.tok_tile));
      for (int i = 0; i < nkb; ++i) {
        const int s = i % S;
        const uint32_t r = static_cast<uint32_t>(i / S);
        if (!mbar_wait(kW4 ? &afull[s] : &full[s], r & 1u, p.wait_ns)) {
          set_error(p.err, DEV_TIMEOUT_MMA);
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        tc_fence_after();
        uint8_t* st = smem + s * p.stage_bytes;
        const uint64_t adesc = sw128_kmajor_desc(smem_u32(st));
        const uint64_t bdesc = sw128_kmajor_desc(smem_u32(st + kATileBytes));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16_ss(tmem_d, adesc + 2 * kk, bdesc + 2 * kk, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
      }
      mma_commit(accum);
    }
  } else {
    const int ct = threadIdx.x - 64;
    if (kW4) {
      const int row = ct >> 1;
      const int hf = ct & 1;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % S;
        const uint32_t r = static_cast<uint32_t>(i / S);
        if (!mbar_wait(&full[s], r & 1u, p.wait_ns)) {
          set_error(p.err, DEV_TIMEOUT_CONSUMER);
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        uint8_t* st = smem + s * p.stage_bytes;
        const uint8_t* raw = st + kATileBytes + b_bytes;
        const uint4 c = *reinterpret_cast<const uint4*>(raw + row * 32 + hf * 16);
        const __half2 mm = *reinterpret_cast<const __half2*>(raw + kTileCodeBytes + row * 4);
        const __half2 m2 = __low2half2(mm);
        const __half2 s2 = __high2half2(mm);
        uint8_t* arow = st + row * 128;
        const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int phys = (hf * 4 + j) ^ (row & 7);
          *reinterpret_cast<uint4*>(arow + phys * 16) = dequant8(words[j], s2, m2);
        }
        fence_proxy_async_smem();
        mbar_arrive(&afull[s]);
      }
    }
    // epilogue
    const bool ok = mbar_wait(accum, 0, p.wait_ns);
    if (!ok) set_error(p.err, DEV_TIMEOUT_EPILOGUE);
    tc_fence_after();
    if (ok && !*abort_flag) {
      const int q = warp & 3;
      const int wg = (warp - 2) >> 2;
      const int feat = n_tile * 128 + q * 32 + lane;
      const bool fvalid = feat < p.n;
      const uint32_t tbase = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
      float bias_v = 0.f;
      if ((p.epi & EPI_BIAS) && fvalid && !p.splitk) bias_v = __half2float(p.bias[feat]);
      const int tok0 = t_tile * p.tok_tile;
      for (int c0 = wg * 16; c0 < p.tok_tile; c0 += 32) {
        uint32_t rr[16];
        tmem_ld_x16(tbase + static_cast<uint32_t>(c0), rr);
        tmem_ld_wait();
        if (!fvalid) continue;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int tok = tok0 + c0 + j;
          if (tok >= p.m) break;
          float v = __uint_as_float(rr[j]);
          if (p.splitk) {
            atomicAdd(p.yf + static_cast<size_t>(tok) * p.ldyf + feat, v);
          } else if (p.epi & EPI_F32_OUT) {
            p.yf[static_cast<size_t>(tok) * p.ldyf + feat] = v;
          } else {
            v += bias_v;
            if (p.epi & EPI_GELU) v = gelu_erf(v);
            if (p.epi & EPI_RESIDUAL)
              v += __half2float(p.residual[static_cast<size_t>(tok) * p.ld_res + feat]);
            p.y[static_cast<size_t>(tok) * p.ldy + feat] = __float2half_rn(v);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // The accumulator barrier completes only when every issued MMA has
    // finished, so TMEM is never released under a running MMA.
    if (lane == 0) mbar_wait(accum, 0, drain_ns(p.wait_ns));
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_d, p.tmem_cols);
  }
}

// Split-K finish: Y = epilogue(sum of partials).
__global__ void splitk_finish_kernel(const float* __restrict__ acc, int m, int n, const __half* bias,
                                     const __half* residual, int ld_res, __half* y, int ldy,
                                     float* yf, int ldyf, int epi) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<size_t>(m) * n) return;
  const int tok = static_cast<int>(idx / n);
  const int feat = static_cast<int>(idx % n);
  float v = acc[idx];
  if (epi & EPI_F32_OUT) {
    yf[static_cast<size_t>(tok) * ldyf + feat] = v;
    return;
  }
  if (epi & EPI_BIAS) v += __half2float(bias[feat]);
  if (epi & EPI_GELU) v = gelu_erf(v);
  if (epi & EPI_RESIDUAL) v += __half2float(residual[static_cast<size_t>(tok) * ld_res + feat]);
  y[static_cast<size_t>(tok) * ldy + feat] = __float2half_rn(v);
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

// 2-D fp16 tensor [rows][cols] with row stride ld (elements), box 64 x box_rows,
// 128-byte swizzle, zero fill out of bounds.
bool make_tmap(CUtensorMap* map, const void* base, int rows, int cols, int ld, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Plan {
  int tok_tile, tok_tiles, n_tiles, splits, kb_per_split, stages;
  uint32_t stage_bytes;
  size_t smem;
};

int round_up(int a, int b) { return (a + b - 1) / b * b; }

Plan make_plan(int m, int n, int k, int w_bits, int force_splits, int force_tok_tile) {
  Plan P{};
  const int kb_total = k / 64;
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
  P.n_tiles = (n + 127) / 128;
  const int tiles = P.n_tiles * P.tok_tiles;
  int splits = 1;
  if (force_splits > 0) {
    splits = force_splits;
  } else {
    const int sms = runtime().num_sms;
    if (tiles < sms) splits = min(max(1, kb_total / 8), (sms + tiles - 1) / tiles);
  }
  splits = max(1, min(splits, kb_total));
  P.kb_per_split = (kb_total + splits - 1) / splits;
  P.splits = (kb_total + P.kb_per_split - 1) / P.kb_per_split;
  P.stage_bytes = static_cast<uint32_t>(kATileBytes + P.tok_tile * 128 + (w_bits == 4 ? kRawBytes : 0));
  P.stages = min(8, static_cast<int>((kMaxSmem - 1024 - kBarrierBytes) / P.stage_bytes));
  P.smem = static_cast<size_t>(P.stages) * P.stage_bytes + 1024 + kBarrierBytes;
  return P;
}

template <bool kW4>
cudaError_t configure_once() {
  static cudaError_t status = cudaErrorNotReady;
  static std::once_flag once;
  std::call_once(once, [] {
    status = cudaFuncSetAttribute(gemm_tc_kernel<kW4>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  });
  return status;
}

}  // namespace

size_t linear_workspace_bytes(int m, int n, int k, int w_bits, int force_splits) {
  const Plan P = make_plan(m, n, k, w_bits, force_splits, 0);
  return P.splits > 1 ? static_cast<size_t>(m) * n * sizeof(float) : 0;
}

cudaError_t launch_linear(const LinearArgs& a, void* ws, size_t ws_bytes, cudaStream_t s) {
  if (a.m == 0 || a.n == 0) return cudaSuccess;
  const Plan P = make_plan(a.m, a.n, a.k, a.w_bits, a.force_splits, a.force_tok_tile);
  const bool w4 = a.w_bits == 4;
  cudaError_t e = w4 ? configure_once<true>() : configure_once<false>();
  if (e != cudaSuccess) return e;
  CUtensorMap tx, tw;
  if (!make_tmap(&tx, a.x, a.m, a.k, a.ldx, P.tok_tile)) return cudaErrorInvalidValue;
  if (w4) {
    tw = tx;
  } else if (!make_tmap(&tw, a.w, a.n, a.k, a.k, 128)) {
    return cudaErrorInvalidValue;
  }
  GemmParams p{};
  p.wq = static_cast<const uint8_t*>(a.w);
  p.m = a.m;
  p.n = a.n;
  p.k = a.k;
  p.kb_total = a.k / 64;
  p.kb_per_split = P.kb_per_split;
  p.tok_tile = P.tok_tile;
  p.stages = P.stages;
  p.stage_bytes = P.stage_bytes;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(P.tok_tile)) cols <<= 1;
  p.tmem_cols = cols;
  p.bias = a.bias;
  p.residual = a.residual;
  p.ld_res = a.ld_res;
  p.epi = a.epi;
  p.wait_ns = runtime().wait_limit_ns;
  p.err = runtime().err;
  const bool split = P.splits > 1;
  if (split) {
    const size_t need = static_cast<size_t>(a.m) * a.n * sizeof(float);
    if (ws == nullptr || ws_bytes < need) return cudaErrorInvalidValue;
    e = cudaMemsetAsync(ws, 0, need, s);
    if (e != cudaSuccess) return e;
    p.splitk = 1;
    p.yf = static_cast<float*>(ws);
    p.ldyf = a.n;
  } else if (a.epi & EPI_F32_OUT) {
    p.yf = static_cast<float*>(a.y);
    p.ldyf = a.ldy;
  } else {
    p.y = static_cast<__half*>(a.y);
    p.ldy = a.ldy;
  }
  dim3 grid(P.n_tiles, P.tok_tiles, P.splits);
  if (w4)
    gemm_tc_kernel<true><<<grid, kThreads, P.smem, s>>>(tx, tw, p);
  else
    gemm_tc_kernel<false><<<grid, kThreads, P.smem, s>>>(tx, tw, p);
  e = launched();
  if (e != cudaSuccess || !split) return e;
  const size_t total = static_cast<size_t>(a.m) * a.n;
  splitk_finish_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(
      static_cast<const float*>(ws), a.m, a.n, a.bias, a.residual, a.ld_res, static_cast<__half*>(a.y),
      a.ldy, static_cast<float*>(a.y), a.ldy, a.epi);
  return launched();
}

}  // namespace flexq

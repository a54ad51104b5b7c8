// Group-wise asymmetric 4-bit codec ("FlexGen研究学术报告", section 三(C):
// groups of 64 contiguous elements, fp16 min and scale per group, 4-bit codes,
// dequantized to fp16 before compute).
//
// Arithmetic (bit-exact by contract): per group, mn/mx = min/max of the fp16
// values with -0 canonicalised to +0; scale = fp16_rn((mx - mn) / 15) with fp32
// round-to-nearest subtract and divide; min = fp16(mn) (exact); code =
// clamp(rint((x - min) / scale), 0, 15) in fp32, or 0 when scale is 0.
// Dequantization is fp16_rn(fp32(code * scale) + min) with no fused
// multiply-add.  Explicit __f*_rn intrinsics keep the compiler from
// contracting anything.
//
// Work split: two lanes per group, 32 elements each (four 16-byte loads), the
// min/max reduced across the lane pair with one shuffle, and each lane's 32
// codes leaving as one coalesced 16-byte store.
#include "kernels.h"
#include "quant_common.cuh"

namespace flexq {
namespace {

__global__ void quantize_kernel(const __half* __restrict__ x, size_t n_groups,
                                uint8_t* __restrict__ codes, __half* __restrict__ mn,
                                __half* __restrict__ sc) {
  const size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t group = t >> 1;
  const int half_id = static_cast<int>(t & 1);
  const bool valid = group < n_groups;
  float v[32];
  load32(x + (valid ? group * 64 + half_id * 32 : 0), v, valid);
  uint32_t q[32];
  __half m16, s16;
  q64_lane_pair(v, q, m16, s16);
  if (!valid) return;
  uint4 out;
  out.x = pack_canonical(q + 0);
  out.y = pack_canonical(q + 8);
  out.z = pack_canonical(q + 16);
  out.w = pack_canonical(q + 24);
  *reinterpret_cast<uint4*>(codes + group * 32 + half_id * 16) = out;
  if (half_id == 0) {
    mn[group] = m16;
    sc[group] = s16;
  }
}

__global__ void dequantize_kernel(const uint8_t* __restrict__ codes, const __half* __restrict__ mn,
                                  const __half* __restrict__ sc, size_t n_groups,
                                  __half* __restrict__ out) {
  const size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t group = t >> 1;
  if (group >= n_groups) return;
  const int half_id = static_cast<int>(t & 1);
  const uint4 c = *reinterpret_cast<const uint4*>(codes + group * 32 + half_id * 16);
  const float s = __half2float(sc[group]);
  const float m = __half2float(mn[group]);
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  __align__(16) __half r[32];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float q = static_cast<float>((w[j] >> (4 * e)) & 0xF);
      r[j * 8 + e] = __float2half_rn(__fadd_rn(__fmul_rn(q, s), m));
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(out + group * 64 + half_id * 32);
#pragma unroll
  for (int j = 0; j < 4; ++j) dst[j] = reinterpret_cast<const uint4*>(r)[j];
}

// Canonical codes (row-major [n][k/2], low nibble = even element) + separate
// min/scale arrays -> the GEMM's tiled layout.  One thread per (row, group).
__global__ void pack_weight_kernel(const uint8_t* __restrict__ codes, const __half* __restrict__ mn,
                                   const __half* __restrict__ sc, int n_out, int k_in, int n_pad,
                                   uint8_t* __restrict__ packed) {
  const int kb_total = k_in / 64;
  const size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<size_t>(n_pad) * kb_total) return;
  const int r = static_cast<int>(t / kb_total);
  const int kb = static_cast<int>(t % kb_total);
  uint8_t* tile = packed + (static_cast<size_t>(r / kTileRows) * kb_total + kb) * kTileBytes;
  const int rr = r % kTileRows;
  uint32_t words[8];
  __half2 meta = __halves2half2(__float2half(0.f), __float2half(0.f));
  if (r < n_out) {
    const uint4* src = reinterpret_cast<const uint4*>(codes + (static_cast<size_t>(r) * k_in + kb * 64) / 2);
    const uint4 a = src[0], b = src[1];
    const uint32_t cw[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t q[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) q[e] = (cw[j] >> (4 * e)) & 0xF;
      words[j] = pack_tiled(q);
    }
    const size_t g = static_cast<size_t>(r) * kb_total + kb;
    meta = __halves2half2(mn[g], sc[g]);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) words[j] = 0;
  }
  uint4* dst = reinterpret_cast<uint4*>(tile + rr * 32);
  dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
  dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
  *reinterpret_cast<__half2*>(tile + kTileCodeBytes + rr * 4) = meta;
}

// fp16 W [n][k] -> tiled 4-bit layout directly (same codes as quantize_kernel).
__global__ void quantize_weight_kernel(const __half* __restrict__ w, int n_out, int k_in, int n_pad,
                                       uint8_t* __restrict__ packed) {
  const int kb_total = k_in / 64;
  const size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t group = t >> 1;
  const int half_id = static_cast<int>(t & 1);
  const bool in_grid = group < static_cast<size_t>(n_pad) * kb_total;
  const int r = in_grid ? static_cast<int>(group / kb_total) : 0;
  const int kb = in_grid ? static_cast<int>(group % kb_total) : 0;
  const bool valid = in_grid && r < n_out;
  float v[32];
  load32(w + (valid ? static_cast<size_t>(r) * k_in + kb * 64 + half_id * 32 : 0), v, valid);
  uint32_t q[32];
  __half m16, s16;
  q64_lane_pair(v, q, m16, s16);
  if (!in_grid) return;
  uint8_t* tile = packed + (static_cast<size_t>(r / kTileRows) * kb_total + kb) * kTileBytes;
  const int rr = r % kTileRows;
  uint4 out = make_uint4(0, 0, 0, 0);
  if (valid) {
    out.x = pack_tiled(q + 0);
    out.y = pack_tiled(q + 8);
    out.z = pack_tiled(q + 16);
    out.w = pack_tiled(q + 24);
  }
  *reinterpret_cast<uint4*>(tile + rr * 32 + half_id * 16) = out;
  if (half_id == 0) {
    const __half2 meta = valid ? __halves2half2(m16, s16)
                               : __halves2half2(__float2half(0.f), __float2half(0.f));
    *reinterpret_cast<__half2*>(tile + kTileCodeBytes + rr * 4) = meta;
  }
}

}  // namespace

cudaError_t launch_quantize(const __half* x, size_t n, uint8_t* codes, __half* mn, __half* sc,
                            cudaStream_t s) {
  const size_t groups = n / 64;
  if (groups == 0) return cudaSuccess;
  const size_t threads = groups * 2;
  quantize_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, s>>>(x, groups, codes, mn,
                                                                               sc);
  return launched();
}

cudaError_t launch_dequantize(const uint8_t* codes, const __half* mn, const __half* sc, size_t n,
                              __half* out, cudaStream_t s) {
  const size_t groups = n / 64;
  if (groups == 0) return cudaSuccess;
  const size_t threads = groups * 2;
  dequantize_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, s>>>(codes, mn, sc,
                                                                                 groups, out);
  return launched();
}

cudaError_t launch_pack_weight(const uint8_t* codes, const __half* mn, const __half* sc, int n_out,
                               int k_in, uint8_t* packed, cudaStream_t s) {
  const int n_pad = (n_out + kTileRows - 1) / kTileRows * kTileRows;
  const size_t threads = static_cast<size_t>(n_pad) * (k_in / 64);
  if (threads == 0) return cudaSuccess;
  pack_weight_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, s>>>(
      codes, mn, sc, n_out, k_in, n_pad, packed);
  return launched();
}

cudaError_t launch_quantize_weight(const __half* w, int n_out, int k_in, uint8_t* packed,
                                   cudaStream_t s) {
  const int n_pad = (n_out + kTileRows - 1) / kTileRows * kTileRows;
  const size_t threads = static_cast<size_t>(n_pad) * (k_in / 64) * 2;
  if (threads == 0) return cudaSuccess;
  quantize_weight_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, s>>>(
      w, n_out, k_in, n_pad, packed);
  return launched();
}

}  // namespace flexq

// KV-cache append: the decode update x_K <- Concat(x_K, t W_K) (likewise V),
// along the sequence axis ("FlexGen: High-Throughput Generative Inference ..."
// walk-through, section "P/D阶段计算", decoding phase), and the prefill's bulk
// write of slots 0..s-1.  In 4-bit mode each (sequence, head, token) row of d
// elements is quantized on the way in with the group-wise format of
// "FlexGen研究学术报告" section 三(C) (groups of 64 along the head dimension, so
// d in {64, 128} never straddles heads); in 16-bit mode the fp16 row is copied.
//
// Cache layout per layer: K and V each [b][heads][max_len][d/2] bytes of codes
// (low nibble = even element) plus [b][heads][max_len][d/64] (min, scale) fp16
// pairs; 16-bit: [b][heads][max_len][d] fp16.
#include "kernels.h"
#include "quant_common.cuh"

namespace flexq {
namespace {

// grid.y selects K (0) or V (1).  Two lanes per 64-element group.
__global__ void kv_append_q4_kernel(const __half* __restrict__ k_src, const __half* __restrict__ v_src,
                                    int ld_src, int b, int ntok, int heads, int d, KvView kv, int pos0) {
  const bool is_v = blockIdx.y == 1;
  const __half* src = is_v ? v_src : k_src;
  uint8_t* codes = static_cast<uint8_t*>(is_v ? kv.v : kv.k);
  __half2* meta = static_cast<__half2*>(is_v ? kv.v_meta : kv.k_meta);
  const int gpr = d / 64;  // groups per head row
  const size_t n_groups = static_cast<size_t>(b) * ntok * heads * gpr;
  const size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t g = t >> 1;
  const int half_id = static_cast<int>(t & 1);
  const bool valid = g < n_groups;
  const int gd = valid ? static_cast<int>(g % gpr) : 0;
  const size_t rest = valid ? g / gpr : 0;
  const int j = static_cast<int>(rest % heads);
  const size_t row = rest / heads;  // i * ntok + tt
  const int tt = static_cast<int>(row % ntok);
  const int i = static_cast<int>(row / ntok);
  float v[32];
  load32(src + (valid ? row * ld_src + static_cast<size_t>(j) * d + gd * 64 + half_id * 32 : 0), v,
         valid);
  uint32_t q[32];
  __half m16, s16;
  q64_lane_pair(v, q, m16, s16);
  if (!valid) return;
  const size_t slot = (static_cast<size_t>(i) * heads + j) * kv.max_len + pos0 + tt;
  uint4 out;
  out.x = pack_canonical(q + 0);
  out.y = pack_canonical(q + 8);
  out.z = pack_canonical(q + 16);
  out.w = pack_canonical(q + 24);
  *reinterpret_cast<uint4*>(codes + slot * (d / 2) + gd * 32 + half_id * 16) = out;
  if (half_id == 0) meta[slot * gpr + gd] = __halves2half2(m16, s16);
}

__global__ void kv_append_f16_kernel(const __half* __restrict__ k_src, const __half* __restrict__ v_src,
                                     int ld_src, int b, int ntok, int heads, int d, KvView kv,
                                     int pos0) {
  const bool is_v = blockIdx.y == 1;
  const __half* src = is_v ? v_src : k_src;
  __half* dst = static_cast<__half*>(is_v ? kv.v : kv.k);
  const int vpr = d / 8;  // 16-byte vectors per head row
  const size_t n_vec = static_cast<size_t>(b) * ntok * heads * vpr;
  const size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n_vec) return;
  const int e = static_cast<int>(t % vpr);
  const size_t rest = t / vpr;
  const int j = static_cast<int>(rest % heads);
  const size_t row = rest / heads;
  const int tt = static_cast<int>(row % ntok);
  const int i = static_cast<int>(row / ntok);
  const uint4 val = *reinterpret_cast<const uint4*>(src + row * ld_src + static_cast<size_t>(j) * d + e * 8);
  const size_t slot = (static_cast<size_t>(i) * heads + j) * kv.max_len + pos0 + tt;
  *reinterpret_cast<uint4*>(dst + slot * d + e * 8) = val;
}

}  // namespace

cudaError_t launch_kv_append(const __half* k_src, const __half* v_src, int ld_src, int b, int ntok,
                             int heads, int d, int kv_bits, const KvView& kv, int pos0,
                             cudaStream_t s) {
  if (b == 0 || ntok == 0) return cudaSuccess;
  if (kv_bits == 4) {
    const size_t threads = static_cast<size_t>(b) * ntok * heads * (d / 64) * 2;
    dim3 grid(static_cast<unsigned>((threads + 255) / 256), 2);
    kv_append_q4_kernel<<<grid, 256, 0, s>>>(k_src, v_src, ld_src, b, ntok, heads, d, kv, pos0);
  } else {
    const size_t threads = static_cast<size_t>(b) * ntok * heads * (d / 8);
    dim3 grid(static_cast<unsigned>((threads + 255) / 256), 2);
    kv_append_f16_kernel<<<grid, 256, 0, s>>>(k_src, v_src, ld_src, b, ntok, heads, d, kv, pos0);
  }
  return launched();
}

}  // namespace flexq

// KV-cache append: the decode update x_K <- Concat(x_K, t W_K) (likewise V),
// along the sequence axis ("FlexGen: High-Throughput Generative Inference ..."
// walk-through, section "P/D阶段计算", decoding phase), and the prefill's bulk
// write of slots 0..s-1.  In 4-bit mode each (sequence, head, token) row of d
// elements is quantized on the way in with the group-wise format of
// "FlexGen研究学术报告" section 三(C) (groups of 64 along the head dimension, so
// d in {64, 128} never straddles heads); in 16-bit mode the fp16 row is copied.
//
// 4-bit cache layout per layer and (sequence, head):
//   K codes   [max_len][d/2] bytes, canonical (low nibble = even element);
//   V codes   [pad8(max_len)/8][d] 32-bit words, token-interleaved: nibble k
//             of word (block, e) is the code of token 8*block + k at dimension
//             e, so decode attention can weight 8 tokens of one dimension with
//             integer dot products;
//   K/V meta  [max_len][d/64] (min, scale) fp16 pairs.
// The codes of a row are exactly those flexq_quantize gives the same 64-element
// group; only where V's nibbles are stored differs.
#include "kernels.h"
#include "quant_common.cuh"

namespace flexq {
namespace {

// K rows, canonical layout.  Two lanes per 64-element group.
__global__ void kv_append_k4_kernel(const __half* __restrict__ src, int ld_src, int b, int ntok, int heads, int d,
                                    uint8_t* __restrict__ codes, __half2* __restrict__ meta, int max_len, int pos0) {
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
  load32(src + (valid ? row * ld_src + static_cast<size_t>(j) * d + gd * 64 + half_id * 32 : 0), v, valid);
  uint32_t q[32];
  __half m16, s16;
  q64_lane_pair(v, q, m16, s16);
  if (!valid) return;
  const size_t slot = (static_cast<size_t>(i) * heads + j) * max_len + pos0 + tt;
  uint4 out;
  out.x = pack_canonical(q + 0);
  out.y = pack_canonical(q + 8);
  out.z = pack_canonical(q + 16);
  out.w = pack_canonical(q + 24);
  *reinterpret_cast<uint4*>(codes + slot * (d / 2) + gd * 32 + half_id * 16) = out;
  if (half_id == 0) meta[slot * gpr + gd] = __halves2half2(m16, s16);
}

// V rows of relative tokens [tt0, tt1) into the token-interleaved layout, one
// nibble per (token, dimension).  Words shared with other tokens of the same
// 8-token block are updated with atomics unless a single token is written.
__global__ void kv_append_v4_tokens_kernel(const __half* __restrict__ src, int ld_src, int b, int ntok, int tt0,
                                           int tt1, int heads, int d, uint32_t* __restrict__ words,
                                           __half2* __restrict__ meta, int max_len, int pos0, bool exclusive) {
  const int gpr = d / 64;
  const int span = tt1 - tt0;
  const size_t n_groups = static_cast<size_t>(b) * span * heads * gpr;
  const size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t g = t >> 1;
  const int half_id = static_cast<int>(t & 1);
  const bool valid = g < n_groups;
  const int gd = valid ? static_cast<int>(g % gpr) : 0;
  const size_t rest = valid ? g / gpr : 0;
  const int j = static_cast<int>(rest % heads);
  const size_t r2 = rest / heads;
  const int tt = tt0 + static_cast<int>(r2 % span);
  const int i = static_cast<int>(r2 / span);
  const size_t row = static_cast<size_t>(i) * ntok + tt;
  float v[32];
  load32(src + (valid ? row * ld_src + static_cast<size_t>(j) * d + gd * 64 + half_id * 32 : 0), v, valid);
  uint32_t q[32];
  __half m16, s16;
  q64_lane_pair(v, q, m16, s16);
  if (!valid) return;
  const int slot = pos0 + tt;
  const size_t head_row = static_cast<size_t>(i) * heads + j;
  uint32_t* w = words + (head_row * (kv_pad_len(max_len) / 8) + slot / 8) * d + gd * 64 + half_id * 32;
  const int sh = 4 * (slot & 7);
  const uint32_t clear = ~(0xFu << sh);
  if (exclusive) {
    // the lane owns these 32 words: one 128-byte read-modify-write in 16-byte vectors
    uint4* w4 = reinterpret_cast<uint4*>(w);
    uint4 cur[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) cur[u] = w4[u];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      cur[u].x = (cur[u].x & clear) | (q[4 * u] << sh);
      cur[u].y = (cur[u].y & clear) | (q[4 * u + 1] << sh);
      cur[u].z = (cur[u].z & clear) | (q[4 * u + 2] << sh);
      cur[u].w = (cur[u].w & clear) | (q[4 * u + 3] << sh);
      w4[u] = cur[u];
    }
  } else {
#pragma unroll 4
    for (int e = 0; e < 32; ++e) {
      atomicAnd(w + e, clear);
      atomicOr(w + e, q[e] << sh);
    }
  }
  if (half_id == 0) meta[(head_row * max_len + slot) * gpr + gd] = __halves2half2(m16, s16);
}

// V rows of whole 8-token blocks [blk0, blk0 + nblk) (absolute block index):
// one unit = (sequence, head, block) = 8 tokens x d dimensions, 8 * d / 32
// lanes per unit.  Codes are quantized by lane pairs, transposed through
// shared memory, and each lane stores four finished words.
constexpr int kBlkThreads = 256;
__global__ void __launch_bounds__(kBlkThreads) kv_append_v4_blocks_kernel(
    const __half* __restrict__ src, int ld_src, int b, int ntok, int heads, int d, int blk0, int nblk,
    uint32_t* __restrict__ words, __half2* __restrict__ meta, int max_len, int pos0) {
  __shared__ __align__(16) uint8_t sm[kBlkThreads / 32][8][128];  // up to 8 units (d = 64) share a warp's rows
  const int lanes_per_unit = 8 * d / 32;  // 32 (d = 128) or 16 (d = 64)
  const int units_per_cta = kBlkThreads / lanes_per_unit;
  const size_t n_units = static_cast<size_t>(b) * heads * nblk;
  const size_t unit = static_cast<size_t>(blockIdx.x) * units_per_cta + threadIdx.x / lanes_per_unit;
  const int lu = threadIdx.x % lanes_per_unit;
  const bool valid = unit < n_units;
  const int gh = lu % (d / 32);  // 32-dimension slice of the token row
  const int k = lu / (d / 32);   // token inside the block
  const int blk = valid ? static_cast<int>(unit % nblk) + blk0 : blk0;
  const size_t head_row = valid ? unit / nblk : 0;
  const int j = static_cast<int>(head_row % heads);
  const int i = static_cast<int>(head_row / heads);
  const int slot = blk * 8 + k;
  const int tt = slot - pos0;
  const size_t row = static_cast<size_t>(i) * ntok + tt;
  float v[32];
  load32(src + (valid ? row * ld_src + static_cast<size_t>(j) * d + gh * 32 : 0), v, valid);
  uint32_t q[32];
  __half m16, s16;
  q64_lane_pair(v, q, m16, s16);
  // stage this lane's 32 codes (one byte each) at sm[unit slot][k][dims]
  const int wslot = (threadIdx.x / 32) * (32 / lanes_per_unit) + (threadIdx.x % 32) / lanes_per_unit;
  uint8_t* row_sm = &sm[0][0][0] + (static_cast<size_t>(wslot) * 8 + k) * d + gh * 32;
#pragma unroll
  for (int e = 0; e < 32; e += 4)
    *reinterpret_cast<uint32_t*>(row_sm + e) = q[e] | (q[e + 1] << 8) | (q[e + 2] << 16) | (q[e + 3] << 24);
  __syncwarp();
  if (!valid) return;
  if ((gh & 1) == 0) meta[(head_row * max_len + slot) * (d / 64) + gh / 2] = __halves2half2(m16, s16);
  // lane lu finishes dimensions 4*lu .. 4*lu+3 of the unit
  const uint8_t* base = &sm[0][0][0] + static_cast<size_t>(wslot) * 8 * d + 4 * lu;
  uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t x = *reinterpret_cast<const uint32_t*>(base + kk * d);
#pragma unroll
    for (int e = 0; e < 4; ++e) out[e] |= ((x >> (8 * e)) & 0xFu) << (4 * kk);
  }
  *reinterpret_cast<uint4*>(words + (head_row * (kv_pad_len(max_len) / 8) + blk) * d + 4 * lu) =
      make_uint4(out[0], out[1], out[2], out[3]);
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

unsigned blocks_for(size_t threads, int per) { return static_cast<unsigned>((threads + per - 1) / per); }

}  // namespace

cudaError_t launch_kv_append(const __half* k_src, const __half* v_src, int ld_src, int b, int ntok,
                             int heads, int d, int kv_bits, const KvView& kv, int pos0,
                             cudaStream_t s) {
  if (b == 0 || ntok == 0) return cudaSuccess;
  if (kv_bits != 4) {
    const size_t threads = static_cast<size_t>(b) * ntok * heads * (d / 8);
    dim3 grid(blocks_for(threads, 256), 2);
    kv_append_f16_kernel<<<grid, 256, 0, s>>>(k_src, v_src, ld_src, b, ntok, heads, d, kv, pos0);
    return launched();
  }
  const size_t k_threads = static_cast<size_t>(b) * ntok * heads * (d / 64) * 2;
  kv_append_k4_kernel<<<blocks_for(k_threads, 256), 256, 0, s>>>(
      k_src, ld_src, b, ntok, heads, d, static_cast<uint8_t*>(kv.k), static_cast<__half2*>(kv.k_meta), kv.max_len,
      pos0);
  cudaError_t e = launched();
  if (e != cudaSuccess) return e;
  // V: whole 8-token blocks by transposition, ragged edges token by token
  const int a0 = (pos0 + 7) & ~7;
  const int a1 = (pos0 + ntok) & ~7;
  uint32_t* words = static_cast<uint32_t*>(kv.v);
  __half2* vmeta = static_cast<__half2*>(kv.v_meta);
  const bool exclusive = ntok == 1;
  if (a1 > a0) {
    const int nblk = (a1 - a0) / 8;
    const int lanes_per_unit = 8 * d / 32;
    const size_t units = static_cast<size_t>(b) * heads * nblk;
    kv_append_v4_blocks_kernel<<<blocks_for(units, kBlkThreads / lanes_per_unit), kBlkThreads, 0, s>>>(
        v_src, ld_src, b, ntok, heads, d, a0 / 8, nblk, words, vmeta, kv.max_len, pos0);
    if ((e = launched()) != cudaSuccess) return e;
  }
  const int edges[2][2] = {{0, (a1 > a0 ? a0 : pos0 + ntok) - pos0}, {(a1 > a0 ? a1 : pos0 + ntok) - pos0, ntok}};
  for (const auto& r : edges) {
    if (r[1] <= r[0]) continue;
    const size_t threads = static_cast<size_t>(b) * (r[1] - r[0]) * heads * (d / 64) * 2;
    kv_append_v4_tokens_kernel<<<blocks_for(threads, 256), 256, 0, s>>>(
        v_src, ld_src, b, ntok, r[0], r[1], heads, d, words, vmeta, kv.max_len, pos0, exclusive);
    if ((e = launched()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace flexq

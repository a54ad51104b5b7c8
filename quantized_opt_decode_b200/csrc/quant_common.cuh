// Device-side group quantizer shared by the codec, the weight packer and the
// KV-cache append (one definition so every producer of 4-bit codes agrees
// bit for bit).  Two adjacent lanes own one 64-element group, 32 elements each.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "kernels.h"

namespace flexq {

// Loads 32 consecutive fp16 values (64 B, 16-B aligned) as fp32; zeros when
// !valid.
__device__ __forceinline__ void load32(const __half* p, float (&v)[32], bool valid) {
  if (valid) {
    const uint4* s = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 u = s[j];
      const __half2* h2 = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h2[e]);
        v[j * 8 + 2 * e] = f.x;
        v[j * 8 + 2 * e + 1] = f.y;
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = 0.f;
  }
}

// Quantizes one 64-element group held by a lane pair (lanes 2i and 2i+1 of the
// warp, 32 elements each).  Every lane of the warp must call this.
__device__ __forceinline__ void q64_lane_pair(const float (&v)[32], uint32_t (&q)[32], __half& m16,
                                              __half& s16) {
  float lo = v[0], hi = v[0];
#pragma unroll
  for (int e = 1; e < 32; ++e) {
    lo = fminf(lo, v[e]);
    hi = fmaxf(hi, v[e]);
  }
  lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, 1));
  hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, 1));
  lo = __fadd_rn(lo, 0.0f);  // -0 -> +0
  hi = __fadd_rn(hi, 0.0f);
  s16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
  m16 = __float2half_rn(lo);
  const float s = __half2float(s16);
  const float m = __half2float(m16);
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    float r = 0.0f;
    if (s != 0.0f) r = fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(v[e], m), s)), 0.0f), 15.0f);
    q[e] = static_cast<uint32_t>(r);
  }
}

// 8 codes -> one 32-bit word, nibble e holds element e (low nibble = even
// element of each byte).
__device__ __forceinline__ uint32_t pack_canonical(const uint32_t* q) {
  uint32_t w = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) w |= (q[e] & 0xF) << (4 * e);
  return w;
}

// 8 codes -> one 32-bit word in the GEMM's order: element e sits in nibble
// (e >> 1) + 4 * (e & 1), so (w >> 4i) & 0x000F000F yields elements 2i and 2i+1
// in the two 16-bit halves.
__device__ __forceinline__ uint32_t pack_tiled(const uint32_t* q) {
  uint32_t w = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) w |= (q[e] & 0xF) << (4 * ((e >> 1) + 4 * (e & 1)));
  return w;
}

// Quantize on append of one (sequence i, head j) at decode: the token's K and
// V rows (d fp16 each) go to cache slot app.pos exactly as the append kernels
// write them (K canonical codes, V the token's nibble in each
// token-interleaved word, (min, scale) per 64 elements).  Called by one whole
// warp; lanes 0 .. 2d/64 - 1 hold K (two per group), the next 2d/64 V.
template <int D>
__device__ __forceinline__ void append_row_q4(const AppendRow& app, const KvView& kv, int i, int j, int heads) {
  constexpr int G = D / 64;
  const int lane = threadIdx.x & 31;
  const bool active = lane < 4 * G;
  const bool is_v = lane >= 2 * G;
  const int l2 = is_v ? lane - 2 * G : lane;
  const int gd = l2 >> 1, half_id = l2 & 1;
  const __half* src = (is_v ? app.v : app.k) + static_cast<size_t>(i) * app.ld + j * D + gd * 64 + half_id * 32;
  float v[32];
  load32(src, v, active);
  uint32_t q[32];
  __half m16, s16;
  q64_lane_pair(v, q, m16, s16);
  if (!active) return;
  const size_t hr = static_cast<size_t>(i) * heads + j;
  const size_t slot = hr * kv.max_len + app.pos;
  if (!is_v) {
    const uint4 out = make_uint4(pack_canonical(q), pack_canonical(q + 8), pack_canonical(q + 16),
                                 pack_canonical(q + 24));
    *reinterpret_cast<uint4*>(static_cast<uint8_t*>(kv.k) + slot * (D / 2) + gd * 32 + half_id * 16) = out;
  } else {
    uint4* w4 = reinterpret_cast<uint4*>(static_cast<uint32_t*>(kv.v) +
                                         (hr * (kv_pad_len(kv.max_len) / 8) + app.pos / 8) * D + gd * 64 +
                                         half_id * 32);
    const int sh = 4 * (app.pos & 7);
    const uint32_t clear = ~(0xFu << sh);
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
  }
  if (half_id == 0) static_cast<__half2*>(is_v ? kv.v_meta : kv.k_meta)[slot * G + gd] = __halves2half2(m16, s16);
}

}  // namespace flexq

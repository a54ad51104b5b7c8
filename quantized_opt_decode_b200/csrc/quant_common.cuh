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

// code = clamp(rint(a / s), 0, 15) with a / s the correctly rounded fp32
// quotient, computed without a division in almost every case: r = a * fl(1/s)
// differs from fl(a / s) by less than |r| * 2^-22 (two roundings of relative
// size 2^-24 in r, one in the quotient), so wherever r is farther than
// |r| * 2^-20 (plus 2^-40) from a rounding boundary k + 1/2, both round to
// the same integer k; only a value that close takes the exact quotient.  r - k
// and 1/2 - |r - k| are exact in fp32 (Sterbenz), so the test itself does not
// round.  s > 0.
__device__ __forceinline__ uint32_t q64_code(float a, float s, float inv_s) {
  const float r = __fmul_rn(a, inv_s);
  float k = rintf(r);
  const float margin = __fadd_rn(__fmul_rn(fabsf(r), 0x1p-20f), 0x1p-40f);
  if (fabsf(__fsub_rn(0.5f, fabsf(__fsub_rn(r, k)))) <= margin) k = rintf(__fdiv_rn(a, s));
  return static_cast<uint32_t>(fminf(fmaxf(k, 0.0f), 15.0f));
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
  const float inv_s = s != 0.0f ? __frcp_rn(s) : 0.0f;
#pragma unroll
  for (int e = 0; e < 32; ++e) q[e] = s != 0.0f ? q64_code(__fsub_rn(v[e], m), s, inv_s) : 0u;
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
// token-interleaved word, (min, scale) per 64 elements).  One warp per
// 64-element group: warp w < d/64 takes K group w, the next d/64 warps the V
// groups, two elements per lane (the group's min and max by warp shuffles,
// which give the same values as any other order); warps past 2d/64 return.
// A V warp fetches the token's interleaved words together with its fp16 pair,
// so the two reads overlap.  The caller synchronises before reading the slot.
template <int D>
__device__ __forceinline__ void append_group_q4(const AppendRow& app, const KvView& kv, int i, int j, int heads,
                                                int warp, int lane) {
  constexpr int G = D / 64;
  if (warp >= 2 * G) return;
  const bool is_v = warp >= G;
  const int gd = is_v ? warp - G : warp;
  const size_t hr = static_cast<size_t>(i) * heads + j;
  const size_t slot = hr * kv.max_len + app.pos;
  uint2* vp = nullptr;
  uint2 vold = make_uint2(0u, 0u);
  if (is_v) {
    vp = reinterpret_cast<uint2*>(static_cast<uint32_t*>(kv.v) +
                                  (hr * (kv_pad_len(kv.max_len) / 8) + app.pos / 8) * D + gd * 64 + 2 * lane);
    vold = *vp;
  }
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(
      (is_v ? app.v : app.k) + static_cast<size_t>(i) * app.ld + j * D + gd * 64 + 2 * lane));
  float lo = fminf(f.x, f.y), hi = fmaxf(f.x, f.y);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  lo = __fadd_rn(lo, 0.0f);  // -0 -> +0
  hi = __fadd_rn(hi, 0.0f);
  const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
  const __half m16 = __float2half_rn(lo);
  const float sc = __half2float(s16);
  const float mn = __half2float(m16);
  uint32_t c0 = 0u, c1 = 0u;
  if (sc != 0.0f) {
    c0 = static_cast<uint32_t>(fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(f.x, mn), sc)), 0.0f), 15.0f));
    c1 = static_cast<uint32_t>(fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(f.y, mn), sc)), 0.0f), 15.0f));
  }
  if (!is_v) {
    static_cast<uint8_t*>(kv.k)[slot * (D / 2) + gd * 32 + lane] = static_cast<uint8_t>(c0 | (c1 << 4));
  } else {
    const int sh = 4 * (app.pos & 7);
    const uint32_t clear = ~(0xFu << sh);
    vold.x = (vold.x & clear) | (c0 << sh);
    vold.y = (vold.y & clear) | (c1 << sh);
    *vp = vold;
  }
  if (lane == 0) static_cast<__half2*>(is_v ? kv.v_meta : kv.k_meta)[slot * G + gd] = __halves2half2(m16, s16);
}

}  // namespace flexq

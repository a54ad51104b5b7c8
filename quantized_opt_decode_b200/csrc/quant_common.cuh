// Device-side group quantizer shared by the codec, the weight packer and the
// KV-cache append (one definition so every producer of 4-bit codes agrees
// bit for bit).  Two adjacent lanes own one 64-element group, 32 elements each.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

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

}  // namespace flexq

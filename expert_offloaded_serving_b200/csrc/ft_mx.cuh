// OCP MX (MXFP4) block quantisation on the device: per block of 32 values,
// scale = clamp(biased_exp(amax) - 2, 0, 254) from the exponent bits of amax,
// elements rounded to nearest even onto the e2m1 grid with saturation by
// cvt.rn.satfinite.e2m1x2.f32 (sign kept).
#pragma once

#include "ft_common.cuh"

namespace ft {

__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{ .reg .b8 b; cvt.rn.satfinite.e2m1x2.f32 b, %1, %2; cvt.u32.u8 %0, b; }" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 2^(127 - e) for e in [0, 254]
__device__ __forceinline__ float mx_inv_scale(int e) {
  return e <= 253 ? __uint_as_float((uint32_t)(254 - e) << 23) : __uint_as_float(0x00400000u);
}

__device__ __forceinline__ int mx_scale_byte(float amax) {
  const int be = (int)((__float_as_uint(amax) >> 23) & 0xff);
  return amax == 0.f ? 0 : min(max(be - 2, 0), 254);
}

// Quantise one 32-element block held as 8 float4; returns the scale byte and
// the 16 bytes of codes (element 2i in the low nibble of byte i).
__device__ __forceinline__ uint32_t mx_quant_block(const float4* v, uint4& q) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; i++)
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
  const int e = mx_scale_byte(amax);
  const float s = mx_inv_scale(e);
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const float4 a = v[2 * i], b = v[2 * i + 1];
    w[i] = cvt_e2m1x2(a.x * s, a.y * s) | (cvt_e2m1x2(a.z * s, a.w * s) << 8) | (cvt_e2m1x2(b.x * s, b.y * s) << 16) |
           (cvt_e2m1x2(b.z * s, b.w * s) << 24);
  }
  q = make_uint4(w[0], w[1], w[2], w[3]);
  return (uint32_t)e;
}

}  // namespace ft

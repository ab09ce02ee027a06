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

// ---------------------------------------------------------------------------
// NVFP4 (two-level) quantisation: a per-tensor fp32 scale s = amax / 2688 and
// g = 1 / (6 s); per 16 values an E4M3 block scale e = E4M3(amax_block * g)
// (nearest even, saturating at 448), dq = value(e) * s, r = 1 / dq and codes
// e2m1(v * r).  Every step is one fp32 operation rounded to nearest even.  A
// tensor whose largest magnitude is below 2^-100 quantises to zero (s = 0),
// which keeps g, r and the products finite; a block with dq == 0 has codes 0.
// ---------------------------------------------------------------------------
constexpr float kNvMinAmax = 7.8886090522101181e-31f;  // 2^-100

struct NvScale {
  float s;  // per-tensor scale
  float g;  // 1 / (6 s)
};

__device__ __forceinline__ NvScale nv_tensor_scale(uint32_t amax_bits) {
  const float amax = __uint_as_float(amax_bits);
  NvScale t{0.f, 0.f};
  if (amax >= kNvMinAmax) {
    t.s = __fdiv_rn(amax, 2688.0f);
    t.g = __frcp_rn(__fmul_rn(t.s, 6.0f));
  }
  return t;
}

// E4M3 byte of v >= 0: nearest, ties to even, saturating at 448.
__device__ __forceinline__ uint32_t cvt_e4m3(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.f), "f"(v));
  return r & 0xffu;
}

// Value of a non-negative finite E4M3 byte (exponent bias 7, 3 fraction
// bits; exponent 0 is m * 2^-9).
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
}

// Quantise 16 values: returns the E4M3 scale byte and the 8 bytes of codes
// (element 2i in the low nibble of byte i).
__device__ __forceinline__ uint32_t nv_quant_block16(const float (&v)[16], NvScale t, uint2& q) {
  q = make_uint2(0u, 0u);
  if (t.s == 0.f) return 0u;
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; i++) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t e = cvt_e4m3(__fmul_rn(amax, t.g));
  const float dq = __fmul_rn(e4m3_value(e), t.s);
  if (dq > 0.f) {
    const float r = __frcp_rn(dq);
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; h++) {
      uint32_t acc = 0;
#pragma unroll
      for (int j = 0; j < 4; j++)
        acc |= cvt_e2m1x2(__fmul_rn(v[8 * h + 2 * j], r), __fmul_rn(v[8 * h + 2 * j + 1], r)) << (8 * j);
      w[h] = acc;
    }
    q = make_uint2(w[0], w[1]);
  }
  return e;
}

// Largest magnitude of a thread's values, folded into *out (fp32 bits of a
// non-negative value order like the values): warp maximum, one atomic.
__device__ __forceinline__ void amax_fold(uint32_t m, uint32_t* out) {
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0 && m) atomicMax(out, m);
}

}  // namespace ft

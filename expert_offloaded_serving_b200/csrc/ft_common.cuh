// Shared definitions of the CUDA library: status bits, blob layout, small
// device helpers.  sm_100a only.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ft_moe.h"

namespace ft {

// bits of the device status word
constexpr int kStNonfinite = 1;
constexpr int kStBadId = 2;
constexpr int kStTimeout = 4;
constexpr int kStMissing = 8;   // an expert pointer was NULL at kernel time

__host__ __device__ inline int64_t pad_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// expert weight formats (ft_model_desc.weight_format)
constexpr int kFmtMx = 0;    // MXFP4: e2m1 codes, one UE8M0 scale per 32 elements
constexpr int kFmtNv = 1;    // NVFP4: e2m1 codes, one E4M3 scale per 16 elements, one fp32 scale per matrix
constexpr int kFmtBf16 = 2;  // BF16 weights

struct BlobLayout {
  int64_t wg, wu, wd, wg_sf, wu_sf, wd_sf, used, stride;
  int64_t ts;  // NVFP4: the three fp32 matrix scales (Wg, Wu, Wd); else -1
  int fmt;
};

// Region offsets of one expert blob (see ft_moe.h).
//   MXFP4: codes Wg [I][H/2], Wu [I][H/2], Wd [H][I/2], then UE8M0 scale
//          regions (128-row x 4-block atoms, blocks of 32 along K).
//   NVFP4: the same codes, then E4M3 scale regions in the same atoms with
//          blocks of 16, then three fp32 matrix scales and 4 zero bytes.
//   BF16:  Wg [I][H], Wu [I][H], Wd [H][I] as bf16 (no scales).
// Each padded to a multiple of 256 bytes.
__host__ __device__ inline BlobLayout blob_layout(int H, int I, int fmt = kFmtMx) {
  BlobLayout b;
  b.fmt = fmt;
  b.ts = -1;
  if (fmt == kFmtBf16) {
    b.wg = 0;
    b.wu = 2 * (int64_t)I * H;
    b.wd = 4 * (int64_t)I * H;
    b.used = 6 * (int64_t)I * H;
    b.wg_sf = b.wu_sf = b.wd_sf = b.used;
    b.stride = pad_up(b.used, 256);
    return b;
  }
  const int blk = fmt == kFmtNv ? 16 : 32;
  int64_t gu = (int64_t)I * H / 2;
  b.wg = 0;
  b.wu = gu;
  b.wd = 2 * gu;
  int64_t end = b.wd + (int64_t)H * I / 2;
  int64_t sf_gu = pad_up(I, 128) * pad_up(H / blk, 4);
  int64_t sf_d = pad_up(H, 128) * pad_up(I / blk, 4);
  b.wg_sf = end;
  b.wu_sf = end + sf_gu;
  b.wd_sf = end + 2 * sf_gu;
  b.used = end + 2 * sf_gu + sf_d;
  if (fmt == kFmtNv) {
    b.ts = b.used;
    b.used += 16;
  }
  b.stride = pad_up(b.used, 256);
  return b;
}

// E4M3 byte (no infinities, S.1111.111 = NaN) -> fp32, exact: exponent 0 is
// subnormal m/8 * 2^-6, else (1 + m/8) * 2^(e - 7).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  const uint32_t s = (b >> 7) & 1u, e = (b >> 3) & 15u, m = b & 7u;
  if (e == 15u && m == 7u) return __uint_as_float(0x7fc00000u);
  const uint32_t bits =
      e == 0u ? (m == 0u ? 0u : __float_as_uint((float)m * 0.001953125f)) : (((e + 120u) << 23) | (m << 20));
  return __uint_as_float(bits | (s << 31));
}

// Byte offset of the 4-byte scale word holding blocks 4a..4a+3 of `row` in a
// scale region with `atoms_k` atoms along K (atom = 128 rows x 4 blocks).
// Device buffers the kernels read or write with vector accesses start on a
// 16-byte boundary (every cudaMalloc'd or torch-allocated buffer does); the
// entry points refuse others before any launch.
__host__ __device__ inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

__host__ __device__ __forceinline__ int64_t sf_word(int row, int a, int atoms_k) {
  return ((int64_t)(row >> 7) * atoms_k + a) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4;
}

// UE8M0 byte -> fp32 2^(e-127) (e = 0 -> 2^-127, a subnormal; 255 -> NaN).
__device__ __forceinline__ float ue8m0_to_f32(uint32_t e) {
  return e == 0 ? __uint_as_float(0x00400000u) : (e == 255 ? __uint_as_float(0x7fc00000u) : __uint_as_float(e << 23));
}

// Two e2m1 codes (low byte of v, element 0 in the low nibble) -> f16x2, exact.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t v) {
  uint32_t h2;
  asm("{ .reg .b8 b; cvt.u8.u32 b, %1; cvt.rn.f16x2.e2m1x2 %0, b; }" : "=r"(h2) : "r"(v));
  return h2;
}

__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t h2) {
  __half2 h = *reinterpret_cast<__half2*>(&h2);
  return __half22float2(h);
}

// d = a * b + c on float pairs (sm_100a packed fp32).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  unsigned long long ua, ub, uc, ud;
  ua = ((unsigned long long)__float_as_uint(a.y) << 32) | __float_as_uint(a.x);
  ub = ((unsigned long long)__float_as_uint(b.y) << 32) | __float_as_uint(b.x);
  uc = ((unsigned long long)__float_as_uint(c.y) << 32) | __float_as_uint(c.x);
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(ud) : "l"(ua), "l"(ub), "l"(uc));
  return make_float2(__uint_as_float((uint32_t)ud), __uint_as_float((uint32_t)(ud >> 32)));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

__device__ __forceinline__ void set_status(int* st, int bits) {
  if (st) atomicOr(st, bits);
}

}  // namespace ft

// Activation quantisers of the prefill path.
//
// OCP MX (MXFP4) quantisation of activation rows:
// per block of 32 values along K, scale = clamp(floor(log2 amax) - 2 + 127,
// 0, 254) taken from the exponent bits of amax, elements rounded to nearest
// even onto the e2m1 grid with saturation by the hardware conversion
// cvt.rn.satfinite.e2m1x2.f32.  Scales go to the 128x4 atom layout.
//
// Pages: prefill runs the experts of a whole layer over many tokens while the
// next layer's experts stream in (aipolix.com, paragraph on bandwidth-adaptive
// execution); MXFP4 is the format the pages name for the expert pool
// (jansverre.net, "Hvor raskt kjører modellene?").
#include "ft_common.cuh"
#include "ft_kernels.h"
#include "ft_mx.cuh"

namespace ft {

__global__ void __launch_bounds__(256) k_quant_rows(const float* __restrict__ x, int64_t R, int K,
                                                    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= R) return;
  const int nb = K / 32;
  const int atoms_k = (int)(pad_up(nb, 4) / 4);
  for (int b = lane; b < nb; b += 32) {
    float4 v[8];
    const float4* src = reinterpret_cast<const float4*>(x + row * K + b * 32);
#pragma unroll
    for (int i = 0; i < 8; i++) v[i] = __ldg(src + i);
    uint4 q;
    uint32_t e = mx_quant_block(v, q);
    *reinterpret_cast<uint4*>(codes + row * (K / 2) + b * 16) = q;
    scales[sf_word((int)row, b >> 2, atoms_k) + (b & 3)] = (uint8_t)e;
  }
}

cudaError_t launch_quantize_rows(const float* x, int64_t R, int K, uint8_t* codes, uint8_t* scales, cudaStream_t s) {
  if (R <= 0) return cudaSuccess;
  k_quant_rows<<<(unsigned)((R + 7) / 8), 256, 0, s>>>(x, R, K, codes, scales);
  return cudaGetLastError();
}

// Largest |x| over n fp32 values, folded into *amax (fp32 bits; zeroed by
// the caller).
__global__ void __launch_bounds__(256) k_amax_f32(const float* __restrict__ x, int64_t n, uint32_t* amax) {
  uint32_t m = 0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    m = max(m, __float_as_uint(x[i]) & 0x7fffffffu);
  amax_fold(m, amax);
}

// The same over bf16 values (the fp32 bits of |x|).
__global__ void __launch_bounds__(256) k_amax_bf16(const uint16_t* __restrict__ x, int64_t n, uint32_t* amax) {
  uint32_t m = 0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    m = max(m, ((uint32_t)x[i] & 0x7fffu) << 16);
  amax_fold(m, amax);
}

cudaError_t launch_amax(const void* x, int64_t n, bool bf16, uint32_t* amax, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (n + 255) / 256;
  const unsigned grid = (unsigned)(want < 8 * (int64_t)nsm ? want : 8 * (int64_t)nsm);
  if (bf16) k_amax_bf16<<<grid, 256, 0, s>>>((const uint16_t*)x, n, amax);
  else k_amax_f32<<<grid, 256, 0, s>>>((const float*)x, n, amax);
  return cudaGetLastError();
}

// NVFP4 rows: a warp per row, a lane per 32 values (two blocks of 16).  The
// per-tensor scale comes from *amax; thread 0 of block 0 stores it to
// *scale_out when that is not NULL.
__global__ void __launch_bounds__(256) k_quant_rows_nv(const float* __restrict__ x, int64_t R, int K,
                                                       const uint32_t* __restrict__ amax, uint8_t* __restrict__ codes,
                                                       uint8_t* __restrict__ scales, float* scale_out) {
  const NvScale t = nv_tensor_scale(*amax);
  if (scale_out && blockIdx.x == 0 && threadIdx.x == 0) *scale_out = t.s;
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= R) return;
  const int atoms_k = K / 64;
  for (int b = lane; b < K / 32; b += 32) {
    const float4* src = reinterpret_cast<const float4*>(x + row * K + b * 32);
    float v[2][16];
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const float4 f = __ldg(src + i);
      v[i >> 2][4 * (i & 3)] = f.x;
      v[i >> 2][4 * (i & 3) + 1] = f.y;
      v[i >> 2][4 * (i & 3) + 2] = f.z;
      v[i >> 2][4 * (i & 3) + 3] = f.w;
    }
    uint2 q0, q1;
    const uint32_t e0 = nv_quant_block16(v[0], t, q0), e1 = nv_quant_block16(v[1], t, q1);
    *reinterpret_cast<uint4*>(codes + row * (K / 2) + b * 16) = make_uint4(q0.x, q0.y, q1.x, q1.y);
    // blocks 2b and 2b + 1 share an atom word: bytes (2b) % 4 and (2b) % 4 + 1
    *reinterpret_cast<uint16_t*>(scales + sf_word((int)row, b >> 1, atoms_k) + ((2 * b) & 3)) =
        (uint16_t)(e0 | (e1 << 8));
  }
}

cudaError_t launch_quantize_rows_nv(const float* x, int64_t R, int K, uint32_t* amax, uint8_t* codes,
                                    uint8_t* scales, float* scale_out, cudaStream_t s) {
  cudaError_t e;
  if ((e = cudaMemsetAsync(amax, 0, sizeof(uint32_t), s)) != cudaSuccess) return e;
  if ((e = launch_amax(x, R * K, false, amax, s)) != cudaSuccess) return e;
  const unsigned grid = (unsigned)(R > 0 ? (R + 7) / 8 : 1);  // one block at R == 0 stores the scale
  k_quant_rows_nv<<<grid, 256, 0, s>>>(x, R, K, amax, codes, scales, scale_out);
  return cudaGetLastError();
}

}  // namespace ft

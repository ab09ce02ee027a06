// OCP MX (MXFP4) quantisation of activation rows for the prefill path:
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

}  // namespace ft

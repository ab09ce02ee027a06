// Kernel launchers shared between the kernel files and the runtime.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "ft_common.cuh"

namespace ft {

struct GemvParams {
  const uint16_t* x;  // bf16 [T][H]
  int T, H, I, E, k, n_shared;
  int max_active;               // grid units reserved for routed experts (>= distinct ids)
  const int32_t* offs;          // [E+1]
  const int32_t* perm;          // [T*k]
  const int32_t* inv;           // [T*k]
  const float* w;               // [T*k]
  const int32_t* active;        // [E]
  const int32_t* n_active;      // [1]
  const uint8_t* const* eptr;   // [E + n_shared] blob pointers of the layer
  BlobLayout lay;
  float* h;                     // [T*k + n_shared*T][I]
  uint16_t* out;                // bf16 [T][H]
  int* status;
};

cudaError_t launch_router_logits(const uint16_t* x, const float* wr, int T, int H, int E, float* logits,
                                 cudaStream_t s);
cudaError_t launch_topk(const float* logits, int T, int E, int k, int renorm, int32_t* ids, float* w, int* status,
                        cudaStream_t s);
size_t permute_smem_bytes(int E);
cudaError_t launch_permute(const int32_t* ids, int P, int E, int32_t* offs, int32_t* perm, int32_t* inv,
                           int32_t* active, int32_t* n_active, int32_t* pad_offs, int* status, cudaStream_t s);
// True when the context-free GEMV kernels below take hidden H and
// intermediate I: each K (H or I) is 128, 256, 512 or a multiple of 1024,
// and H <= 14336 (four tokens of fp32 x fit one CTA's shared memory).
bool gemv_shape_ok(int H, int I);
cudaError_t launch_gate_up(const GemvParams& p, cudaStream_t s);
cudaError_t launch_down_combine(const GemvParams& p, cudaStream_t s);
cudaError_t launch_quantize_rows(const float* x, int64_t R, int K, uint8_t* codes, uint8_t* scales, cudaStream_t s);
// Largest |x| over n values (bf16 or fp32), folded into *amax (fp32 bits);
// the caller zeroes *amax first.
cudaError_t launch_amax(const void* x, int64_t n, bool bf16, uint32_t* amax, cudaStream_t s);
// NVFP4 rows: zeroes *amax, takes the largest |x|, quantises; the per-tensor
// scale goes to *scale_out (device) unless NULL.
cudaError_t launch_quantize_rows_nv(const float* x, int64_t R, int K, uint32_t* amax, uint8_t* codes,
                                    uint8_t* scales, float* scale_out, cudaStream_t s);

}  // namespace ft

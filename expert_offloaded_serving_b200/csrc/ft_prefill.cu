// Prefill path (MXFP4 activations): scratch management and the driver of the
// quantise -> grouped GEMM (gate/up + SwiGLU + quantise h) -> grouped GEMM
// (down) -> combine sequence.
#include "ft_common.cuh"
#include "ft_kernels.h"
#include "ft_runtime.h"

namespace ft {

ft_status ensure_prefill_scratch(PrefillScratch& s, const ft_model_desc& d, int max_tokens) {
  if (s.y) return FT_OK;
  const int64_t T = max_tokens, E = d.n_experts, k = d.top_k, S = d.n_shared;
  s.H = d.hidden;
  s.I = d.inter;
  s.max_pairs = T * k + S * T;
  s.max_rows = pad_up(T * k + 127 * E + S * pad_up(T, 128), 128);
  if (cudaMalloc(&s.xq, (size_t)s.max_rows * s.H / 2) != cudaSuccess ||
      cudaMalloc(&s.xq_sf, (size_t)s.max_rows * s.H / 32) != cudaSuccess ||
      cudaMalloc(&s.hq, (size_t)s.max_rows * s.I / 2) != cudaSuccess ||
      cudaMalloc(&s.hq_sf, (size_t)s.max_rows * s.I / 32) != cudaSuccess ||
      cudaMalloc(&s.y, (size_t)s.max_pairs * s.H * sizeof(float)) != cudaSuccess ||
      cudaMalloc(&s.work, (size_t)(4 * (E + S) + 16) * sizeof(int)) != cudaSuccess) {
    free_prefill_scratch(s);
    return FT_ERR_CUDA;
  }
  return FT_OK;
}

void free_prefill_scratch(PrefillScratch& s) {
  cudaFree(s.xq);
  cudaFree(s.xq_sf);
  cudaFree(s.hq);
  cudaFree(s.hq_sf);
  cudaFree(s.y);
  cudaFree(s.work);
  s = PrefillScratch{};
}

cudaError_t run_prefill(PrefillScratch& s, const PrefillArgs& a, cudaStream_t st) {
  (void)s;
  (void)a;
  (void)st;
  return cudaErrorNotSupported;
}

}  // namespace ft

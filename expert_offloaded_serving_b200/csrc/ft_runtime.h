// Runtime-internal declarations shared by the runtime and the prefill path.
#pragma once

#include <cuda.h>
#include <cstdint>
#include <cuda_runtime.h>

#include "ft_common.cuh"

namespace ft {

constexpr int kDecodeMaxTokens = 16;               // largest T of the decode GEMV path
constexpr size_t kArenaChunkBytes = 256ull << 20;  // physical chunk under the slot arena
constexpr double kHostWaitSeconds = 30.0;          // bounded host waits
constexpr double kHostSpinSeconds = 2e-3;          // ... polled without sleeping for this long first
constexpr int64_t kTraceMaxEvents = 1ll << 22;     // cache events kept between two trace reads

struct PrefillArgs {
  const uint16_t* x;  // bf16 [T][H]
  int T, H, I, E, k, n_shared;
  const int32_t* ids;       // [T*k]
  const float* w;           // [T*k]
  const int32_t* offs;      // [E+1]
  const int32_t* perm;      // [T*k]
  const int32_t* inv;       // [T*k]
  const int32_t* pad_offs;  // [E+1] 128-padded segment starts
  const uint8_t* const* eptr;
  const uint8_t* pool;      // blob 0 of the layer pool (blobs contiguous at lay.stride)
  BlobLayout lay;
  uint16_t* out;  // bf16 [T][H]
  int* status;
};

struct PrefillScratch {
  int64_t max_rows = 0;     // padded activation rows
  int64_t max_pairs = 0;    // rows of y
  int H = 0, I = 0;
  uint8_t* xq = nullptr;    // [max_rows][H/2]
  uint8_t* xq_sf = nullptr; // atoms over [max_rows][H/32] (NVFP4: H/16)
  uint8_t* hq = nullptr;    // [max_rows][I/2]
  uint8_t* hq_sf = nullptr; // atoms over [max_rows][I/32] (NVFP4: I/16)
  float* y = nullptr;       // [max_pairs][H]
  int fmt = 0;              // kFmtMx or kFmtNv (the context's weight format)
  float* hf = nullptr;      // NVFP4: h in fp32 [max_rows][I] before its quantisation
  uint32_t* amax = nullptr; // NVFP4: largest |x| and |h| (fp32 bits)
  CUtensorMap map_xq;       // TMA maps of xq and hq (token side of the GEMMs)
  CUtensorMap map_hq;
};

// Set the message ft_last_error() returns on this thread.
void set_last_error(const char* msg);

int64_t prefill_rows_bound(int T, int E, int k, int n_shared);
ft_status ensure_prefill_scratch(PrefillScratch& s, const ft_model_desc& d, int max_tokens);
void free_prefill_scratch(PrefillScratch& s);
cudaError_t launch_shared_segments(int32_t* pad_offs, int E, int T, int n_shared, cudaStream_t st);
cudaError_t launch_quant_x(const PrefillScratch& s, const PrefillArgs& a, cudaStream_t st);
// NVFP4: quantise the fp32 h the gate/up GEMM left (no-op for MXFP4)
cudaError_t launch_quant_h(const PrefillScratch& s, const PrefillArgs& a, cudaStream_t st);
// mode 0: gate/up GEMM + SwiGLU + MXFP4 h (NVFP4: fp32 h and its largest
// magnitude);  mode 1: down GEMM -> y
cudaError_t launch_prefill_gemm(const PrefillScratch& s, const PrefillArgs& a, int mode, cudaStream_t st);
cudaError_t launch_prefill_combine(const PrefillScratch& s, const PrefillArgs& a, cudaStream_t st);

}  // namespace ft

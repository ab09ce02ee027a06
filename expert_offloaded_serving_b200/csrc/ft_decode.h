// Small-batch decode kernels (fused routing, bulk-staged FP4 GEMV, cluster
// split-K reduction, programmatic dependent launch).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "ft_common.cuh"

namespace ft {

struct DecodeArgs {
  const uint16_t* x;       // bf16 [T][H]
  const float* logits;     // fp32 [T][E]
  int T, H, I, E, k, n_shared, renorm;
  int max_units;           // routed unit slots: min(E, T*k)
  int s_gu, s_dn;          // cluster sizes (K-slices) of gate/up and down
  const uint8_t* const* eptr;  // [E + n_shared] blob pointers
  BlobLayout lay;
  float* h;                // [T*k + n_shared*T][I]
  float* y;                // [T*k + n_shared*T][H]
  uint16_t* out;           // bf16 [T][H]
  int32_t* ids_out;        // [T*k] or NULL (written by one CTA)
  float* w_out;            // [T*k] or NULL
  int* counters;           // [(H/128) * s_dn], zero before the first launch
  int* status;
};

int choose_slices(int K);
size_t decode_smem_bytes(int K, int S, int nmat, int T);
// pdl: launch as a programmatic dependent of the previous kernel in the
// stream.  The gate/up kernel reads its routing inputs (logits, pointer table)
// before griddepcontrol.wait, so it may only be launched that way when those
// inputs were complete before the previous kernel started; the down kernel
// reads nothing produced by gate/up before its wait.
cudaError_t launch_dec_gate_up(const DecodeArgs& a, bool pdl, cudaStream_t s);
cudaError_t launch_dec_down(const DecodeArgs& a, bool pdl, cudaStream_t s);

}  // namespace ft

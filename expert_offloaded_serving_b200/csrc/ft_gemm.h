// Prefill grouped GEMM on tcgen05 block-scaled FP4 MMA (kind::mxf4 for MXFP4,
// kind::mxf4nvf4 for NVFP4).
#pragma once

#include <cuda.h>
#include <cstdint>
#include <cuda_runtime.h>

#include "ft_common.cuh"

namespace ft {

constexpr int kGemmBM = 128;   // weight rows per tile (MMA M)
constexpr int kGemmBN = 128;   // token rows per tile (MMA N)
constexpr int kGemmBK = 256;   // elements of K per pipeline stage (two scale atoms)

// One grouped GEMM: for every 128-row token tile j of the padded activation
// rows (each tile inside one expert's segment) and every 128-row weight tile
// m:  D[m rows][tokens] = W_e[m rows][K] . Xq[tokens][K]^T  (MXFP4 x MXFP4,
// fp32 accumulate in tensor memory), then the epilogue.
struct GemmArgs {
  int K;                     // contraction length (elements), multiple of 256
  int M;                     // weight rows (I for gate/up, H for down)
  int n_tiles_max;           // grid bound on token tiles
  int n_segments;            // E + n_shared
  const int32_t* pad_offs;   // [n_segments + 1] 128-padded row starts
  const int32_t* offs;       // [E + 1] pair offsets (for the down epilogue)
  int T, k, E;
  int64_t blob_stride;       // bytes between consecutive blobs of the pool
  int64_t sfa_off[2];        // scale-region offsets inside a blob (gate, up) or (down)
  const uint8_t* pool;       // blob 0 of the layer pool
  const uint8_t* sfb;        // activation scales, atoms over padded rows
  int mode;                  // 0: gate/up -> SwiGLU -> MXFP4 h;  1: down -> fp32 y
  int fmt;                   // kFmtMx: UE8M0 per 32, kind::mxf4;  kFmtNv: E4M3 per 16, kind::mxf4nvf4
  // NVFP4: each blob's fp32 matrix scales (Wg, Wu, Wd) at ts_off; the
  // activation operand's per-tensor scale from its largest magnitude
  // *amax_in; gate/up writes h in fp32 to hf ([rows][M]) and folds its
  // largest magnitude into *amax_out instead of quantising h
  int64_t ts_off;
  const uint32_t* amax_in;
  uint32_t* amax_out;
  float* hf;
  // gate/up epilogue
  uint8_t* hq;               // [rows][M/2] codes
  uint8_t* hq_sf;            // atoms over [rows][M/32]
  // down epilogue
  float* y;                  // [T*k + n_shared*T][M]
  int* status;
};

struct GemmMaps {
  CUtensorMap a[2];   // weights: (K/2 bytes, M rows, blob) 3-D, 128B swizzle
  CUtensorMap b;      // activations: (K/2 bytes, rows) 2-D, 128B swizzle
};

// Host: encode a tensor map (driver entry point, no libcuda link).
ft_status encode_tmap_3d(CUtensorMap* map, const void* base, uint64_t inner_bytes, uint64_t rows, uint64_t depth,
                         uint64_t row_pitch, uint64_t depth_pitch);
ft_status encode_tmap_2d(CUtensorMap* map, const void* base, uint64_t inner_bytes, uint64_t rows, uint64_t row_pitch);

size_t gemm_smem_bytes(int mode, int fmt);
cudaError_t launch_gemm(const GemmArgs& a, const GemmMaps& maps, cudaStream_t s);

}  // namespace ft

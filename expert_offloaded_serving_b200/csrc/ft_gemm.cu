// Prefill grouped GEMM on the 5th-generation tensor cores: tcgen05.mma
// kind::mxf4 block-scaled (e2m1 x e2m1, UE8M0 per 32 elements), fp32
// accumulators in tensor memory.
//
// Swap-AB: weights are the M = 128 side (rows of Wg/Wu or Wd), tokens the
// N = 128 side, so experts with ~100 tokens fill an MMA without padding the
// large weight dimension.  Per CTA (128 weight rows x 128 padded token rows of
// one expert):
//   warp 0, one thread   TMA loads of the K-stage tiles (128B-swizzled,
//                        cp.async.bulk.tensor) and bulk copies of the matching
//                        scale atoms, on a ring of kStages shared-memory stages
//   warp 1, one thread   tcgen05.cp of the scale atoms into tensor memory and
//                        tcgen05.mma (K = 64 per instruction); tcgen05.commit
//                        frees a stage and finally signals the accumulators
//   warps 0..15          epilogue from tensor memory (tcgen05.ld): warp w reads
//                        TMEM lanes 32(w%4).. (its weight rows) and every
//                        fourth 16-column group of tokens from 16(w/4): SwiGLU
//                        and MXFP4 quantisation of h (gate/up), or fp32 y (down)
// All mbarrier waits are bounded; on a timeout the CTA records the TIMEOUT
// status, stops issuing, waits (bounded) for its copies still in flight, frees
// its tensor memory and returns.
//
// Pages: prefill computes a whole layer's experts over many tokens while the
// next layer's experts cross PCIe (aipolix.com, paragraph on bandwidth-
// adaptive execution; jansverre.net, "Hvorfor er båndbredden viktigere enn
// antall kjerner?"); MXFP4 experts (jansverre.net, "Hvor raskt kjører
// modellene?").
#include "ft_common.cuh"
#include "ft_gemm.h"
#include "ft_mx.cuh"
#include "ft_tc.cuh"

namespace ft {
using namespace tc;
namespace {

constexpr int kThreads = 512;    // 16 warps: warps w, w+4, w+8, w+12 share TMEM lanes 32(w%4).. in the epilogue
constexpr int kEpiGroups = kThreads / 128;  // column groups of the epilogue
constexpr int kStagesGU = 3;     // gate/up: 2 weight tiles + 1 token tile per stage
constexpr int kStagesDn = 4;     // down: 1 + 1
constexpr int kTileBytes = kGemmBM * kGemmBK / 2;   // 16 KB of e2m1 codes
constexpr int kSfBytes = 1024;                      // two 512-byte scale atoms
constexpr int kTmemCols = 512;

// ---------------------------------------------------------------------------
// the kernel.  MODE 0: gate/up (two weight matrices, SwiGLU, MXFP4 h);
// MODE 1: down (one weight matrix, fp32 y).
// ---------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) k_gemm(const __grid_constant__ GemmArgs a,
                                                      const __grid_constant__ GemmMaps maps) {
  constexpr int S = MODE == 0 ? kStagesGU : kStagesDn;
  constexpr int NA = MODE == 0 ? 2 : 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tileA = smem;                              // [S][NA] 16 KB, 1024-aligned
  uint8_t* tileB = tileA + S * NA * kTileBytes;       // [S] 16 KB
  uint8_t* sfA = tileB + S * kTileBytes;              // [S][NA] 1 KB
  uint8_t* sfB = sfA + S * NA * kSfBytes;             // [S] 1 KB
  uint64_t* full = reinterpret_cast<uint64_t*>(sfB + S * kSfBytes);
  uint64_t* empty = full + S;
  uint64_t* accb = empty + S;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accb + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x, jt = blockIdx.y;
  const int row0 = jt * kGemmBN;
  if (row0 >= a.pad_offs[a.n_segments]) return;
  // expert segment holding this token tile (segments are 128-row aligned)
  int lo = 0, hi = a.n_segments - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.pad_offs[mid] <= row0) lo = mid; else hi = mid - 1;
  }
  const int e = lo;
  const int KT = a.K / kGemmBK;
  const int atoms_k = a.K / 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accb, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s_u32(tmem_holder)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t d0 = tmem;                 // accumulator of matrix 0: columns [0, 128)
  const uint32_t d1 = tmem + kGemmBN;       // accumulator of matrix 1: [128, 256)
  const uint32_t sf0 = tmem + 2 * kGemmBN;  // per stage 24 scale columns: A0 +0, A1 +8, B +16

  if (warp == 0 && lane == 0) {
    // ---- producer ----
    const uint8_t* blob = a.pool + (int64_t)e * a.blob_stride;
    const uint32_t bytes = (NA + 1) * (kTileBytes + kSfBytes);
    int issued = 0;  // K stages whose copies went out
    for (int kt = 0; kt < KT; kt++) {
      const int s = kt % S;
      if (kt >= S && !mbar_wait(&empty[s], ((kt / S) - 1) & 1)) {
        set_status(a.status, kStTimeout);
        break;
      }
      mbar_expect(&full[s], bytes);
#pragma unroll
      for (int q = 0; q < NA; q++) {
        tma_3d(tileA + (s * NA + q) * kTileBytes, &maps.a[q], kt * (kGemmBK / 2), mt * kGemmBM, e, &full[s]);
        bulk_g2s(sfA + (s * NA + q) * kSfBytes, blob + a.sfa_off[q] + ((int64_t)mt * atoms_k + 2 * kt) * 512,
                 kSfBytes, &full[s]);
      }
      tma_2d(tileB + s * kTileBytes, &maps.b, kt * (kGemmBK / 2), row0, &full[s]);
      bulk_g2s(sfB + s * kSfBytes, a.sfb + ((int64_t)jt * atoms_k + 2 * kt) * 512, kSfBytes, &full[s]);
      issued = kt + 1;
    }
    // No copy may still be writing this CTA's shared memory when it exits,
    // also after a timeout of either role.  A stage is reissued only after
    // the MMA consumed its previous round, so only the last S issued stages
    // can be in flight; without a timeout the MMA thread has waited for the
    // same phases, so these waits succeed at once.
    for (int kt = issued > S ? issued - S : 0; kt < issued; kt++) mbar_wait(&full[kt % S], (kt / S) & 1);
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer ----
    for (int kt = 0; kt < KT; kt++) {
      const int s = kt % S;
      if (!mbar_wait(&full[s], (kt / S) & 1)) {
        set_status(a.status, kStTimeout);
        break;
      }
      tc_fence_after();
      const uint32_t sfs = sf0 + s * 24;
#pragma unroll
      for (int q = 0; q < NA; q++)
#pragma unroll
        for (int at = 0; at < 2; at++) utccp_32x128(sfs + q * 8 + 4 * at, desc_sf(sfA + (s * NA + q) * kSfBytes + at * 512));
#pragma unroll
      for (int at = 0; at < 2; at++) utccp_32x128(sfs + 16 + 4 * at, desc_sf(sfB + s * kSfBytes + at * 512));
      const uint64_t bd = desc_sw128(tileB + s * kTileBytes);
#pragma unroll
      for (int kk = 0; kk < kGemmBK / 64; kk++) {
        const uint32_t byte = 2u * (kk & 1), col = 4u * (kk >> 1);
        const uint32_t idesc = idesc_mxf4(byte, byte, kGemmBM, kGemmBN);
#pragma unroll
        for (int q = 0; q < NA; q++) {
          const uint64_t ad = desc_sw128(tileA + (s * NA + q) * kTileBytes) + (uint64_t)(kk * 2);  // +32 bytes of K
          mma_mxf4(q == 0 ? d0 : d1, ad, bd + (uint64_t)(kk * 2), idesc, (sfs + q * 8 + col) | (byte << 30),
                   (sfs + 16 + col) | (byte << 30), (kt | kk) != 0 ? 1u : 0u);
        }
      }
      umma_commit(&empty[s]);
    }
    umma_commit(accb);
  }
  __syncwarp();

  // ---- epilogue: warp w owns TMEM lanes 32(w%4).. = weight rows and the
  // token columns 16 * (w/4 + kEpiGroups * j) ----
  const bool have = mbar_wait_warp(accb, 0);
  if (!have && threadIdx.x == 0) set_status(a.status, kStTimeout);
  const int quad = warp & 3, cg = warp >> 2;
  if (have) {
    tc_fence_after();
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    if (MODE == 0) {
      const int I = a.M;
      const int irow = mt * kGemmBM + quad * 32 + lane;
      const int atoms_i = I / 128;
      for (int c0 = 16 * cg; c0 < kGemmBN; c0 += 16 * kEpiGroups) {
        float g[16], u[16];
        tmem_ld16(d0 + lane_off + c0, g);
        tmem_ld16(d1 + lane_off + c0, u);
#pragma unroll
        for (int q = 0; q < 16; q++) {
          const int p = row0 + c0 + q;
          const float hv = silu(g[q]) * u[q];
          float amax = fabsf(hv);
#pragma unroll
          for (int d = 16; d >= 1; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
          const int e8 = mx_scale_byte(amax);
          const float v = hv * mx_inv_scale(e8);
          const float nb = __shfl_xor_sync(0xffffffffu, v, 1);
          if ((lane & 1) == 0) a.hq[(size_t)p * (I / 2) + (irow >> 1)] = (uint8_t)cvt_e2m1x2(v, nb);
          if (lane == 0) a.hq_sf[sf_word(p, mt, atoms_i) + quad] = (uint8_t)e8;
        }
      }
    } else {
      const int H = a.M;
      const int hrow = mt * kGemmBM + quad * 32 + lane;
      const bool shared = e >= a.E;
      const int valid = shared ? a.T : a.offs[e + 1] - a.offs[e];
      const int base_pos = shared ? a.T * a.k + (e - a.E) * a.T : a.offs[e];
      const int r0 = row0 - a.pad_offs[e];
      for (int c0 = 16 * cg; c0 < kGemmBN; c0 += 16 * kEpiGroups) {
        float v[16];
        tmem_ld16(d0 + lane_off + c0, v);
#pragma unroll
        for (int q = 0; q < 16; q++) {
          const int r = r0 + c0 + q;
          if (r < valid) a.y[(size_t)(base_pos + r) * H + hrow] = v[q];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

size_t gemm_smem_bytes(int mode) {
  const int S = mode == 0 ? kStagesGU : kStagesDn, NA = mode == 0 ? 2 : 1;
  return 1024 + (size_t)S * (NA + 1) * (kTileBytes + kSfBytes) + (2 * S + 1) * 8 + 16;
}

cudaError_t launch_gemm(const GemmArgs& a, const GemmMaps& maps, cudaStream_t s) {
  dim3 grid(a.M / kGemmBM, a.n_tiles_max);
  if (a.n_tiles_max <= 0) return cudaSuccess;
  if (a.mode == 0) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem_bytes(0));
    if (e != cudaSuccess) return e;
    k_gemm<0><<<grid, kThreads, gemm_smem_bytes(0), s>>>(a, maps);
  } else {
    cudaError_t e = cudaFuncSetAttribute(k_gemm<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem_bytes(1));
    if (e != cudaSuccess) return e;
    k_gemm<1><<<grid, kThreads, gemm_smem_bytes(1), s>>>(a, maps);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// tensor maps (driver entry point looked up once)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

ft_status encode_tmap_3d(CUtensorMap* map, const void* base, uint64_t inner_bytes, uint64_t rows, uint64_t depth,
                         uint64_t row_pitch, uint64_t depth_pitch) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FT_ERR_CUDA;
  cuuint64_t dims[3] = {inner_bytes, rows, depth};
  cuuint64_t strides[2] = {row_pitch, depth_pitch};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FT_OK : FT_ERR_CUDA;
}

ft_status encode_tmap_2d(CUtensorMap* map, const void* base, uint64_t inner_bytes, uint64_t rows, uint64_t row_pitch) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FT_ERR_CUDA;
  cuuint64_t dims[2] = {inner_bytes, rows};
  cuuint64_t strides[1] = {row_pitch};
  cuuint32_t box[2] = {128, 128};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FT_OK : FT_ERR_CUDA;
}

}  // namespace ft

// Prefill grouped GEMM on the 5th-generation tensor cores: tcgen05.mma
// kind::mxf4 block-scaled (e2m1 x e2m1, UE8M0 per 32 elements), fp32
// accumulators in tensor memory.
//
// Swap-AB: weights are the M = 128 side (rows of Wg/Wu or Wd), tokens the
// N = 128 side, so experts with ~100 tokens fill an MMA without padding the
// large weight dimension.  A tile is (128 weight rows) x (128 padded token
// rows of one expert).
//
// Persistent: one CTA per SM walks the tiles i = CTA, CTA + grid, ...; tile i
// is token tile i / (M/128) and weight tile i % (M/128), so the CTAs running
// at the same time share a few token tiles and the weight tiles of one or two
// experts through L2.  Roles, one CTA of 18 warps:
//   warp 0, one thread   TMA loads of the K-stage tiles (128B-swizzled,
//                        cp.async.bulk.tensor) and bulk copies of the matching
//                        scale atoms into a ring of kStages shared-memory
//                        stages; it runs ahead across tile boundaries
//   warp 1, one thread   tcgen05.cp of the scale atoms into tensor memory and
//                        tcgen05.mma (K = 64 per instruction); tcgen05.commit
//                        frees a stage, and marks a tile's accumulators full
//   warps 2..17          epilogue: warp w reads TMEM lanes 32(w%4).. (its 32
//                        weight rows) and 32 token columns from
//                        32((w-2)/4), frees the accumulators as soon as its
//                        values are in registers, then SwiGLU and MXFP4
//                        quantisation of h (gate/up), or fp32 y (down)
// The down GEMM double-buffers its accumulator in tensor memory; gate/up (two
// 128-column accumulators) has one buffer, which its epilogue releases right
// after the tensor-memory loads, so the next tile's MMAs wait only for those
// loads.  All mbarrier waits are bounded; on a timeout the CTA records the
// TIMEOUT status, stops issuing, waits (bounded) for its copies and tensor
// operations still in flight, frees its tensor memory and returns.
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

constexpr int kWarps = 18;                 // producer, MMA issuer, 16 epilogue warps
constexpr int kThreads = 32 * kWarps;
constexpr int kEpiWarp0 = 2;               // first epilogue warp
constexpr int kEpiWarps = kWarps - kEpiWarp0;
constexpr int kStagesGU = 4;     // gate/up: 2 weight tiles + 1 token tile per stage (51 KB)
constexpr int kStagesDn = 6;     // down: 1 + 1 (34 KB)
constexpr int kTileBytes = kGemmBM * kGemmBK / 2;   // 16 KB of e2m1 codes
// Scale atoms (512 bytes: 128 rows x 4 blocks) per operand and stage of
// kGemmBK elements: 2 for MXFP4 (blocks of 32), 4 for NVFP4 (blocks of 16).
__host__ __device__ constexpr int atoms_per_stage(int fmt) { return fmt == kFmtNv ? 4 : 2; }
constexpr int kTmemCols = 512;
constexpr int kAccCols = 2 * kGemmBN;               // accumulator columns: gate + up, or two down buffers

__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(s_u32(b)) : "memory");
}

// 16 columns of 32-bit TMEM values of this warp's lanes, without the wait.
__device__ __forceinline__ void tmem_ld16_async(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// Wait for this thread's tensor-memory loads; the registers are tied to the
// wait so that no use of them moves above it.
__device__ __forceinline__ void tmem_wait16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

// Lane-wise unsigned maximum of two 16-bit halves.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Expert segment holding padded token row row0 (segments are 128-row aligned).
__device__ __forceinline__ int segment_of(const GemmArgs& a, int row0) {
  int lo = 0, hi = a.n_segments - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.pad_offs[mid] <= row0) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---------------------------------------------------------------------------
// the kernel.  MODE 0: gate/up (two weight matrices, SwiGLU, MXFP4 h);
// MODE 1: down (one weight matrix, fp32 y).
// ---------------------------------------------------------------------------
template <int MODE, int FMT>
__global__ void __launch_bounds__(kThreads, 1) k_gemm(const __grid_constant__ GemmArgs a,
                                                      const __grid_constant__ GemmMaps maps) {
  constexpr int S = MODE == 0 ? kStagesGU : kStagesDn;
  constexpr int NA = MODE == 0 ? 2 : 1;
  constexpr int NB = MODE == 0 ? 1 : 2;   // accumulator buffers
  constexpr int APS = atoms_per_stage(FMT);
  constexpr int kSfBytes = APS * 512;     // scale bytes per operand and stage
  constexpr int SFC = 4 * APS * (NA + 1); // scale columns per stage (4 a tcgen05.cp atom)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tileA = smem;                              // [S][NA] 16 KB, 1024-aligned
  uint8_t* tileB = tileA + S * NA * kTileBytes;       // [S] 16 KB
  uint8_t* sfA = tileB + S * kTileBytes;              // [S][NA] 1 KB
  uint8_t* sfB = sfA + S * NA * kSfBytes;             // [S] 1 KB
  uint64_t* full = reinterpret_cast<uint64_t*>(sfB + S * kSfBytes);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;                     // [NB] MMA -> epilogue
  uint64_t* acc_empty = acc_full + NB;                // [NB] epilogue (one arrive per warp) -> MMA
  uint64_t* fin = acc_empty + NB;                     // the MMA thread's last operations
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_mt = a.M / kGemmBM;
  const int n_jt = min(a.n_tiles_max, a.pad_offs[a.n_segments] / kGemmBN);
  const int n_tiles = n_mt * n_jt;
  if ((int)blockIdx.x >= n_tiles) return;  // the whole CTA, before any barrier or allocation
  const int KT = a.K / kGemmBK;
  const int atoms_k = a.K * APS / kGemmBK;  // scale atoms along K

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NB; b++) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
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
  const uint32_t sf0 = tmem + kAccCols;  // per stage SFC scale columns: A0 +0, A1 +8 (gate/up), B +8*NA

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer ----
      const uint32_t bytes = (NA + 1) * (kTileBytes + kSfBytes);
      int issued = 0;  // K stages whose copies went out, over all tiles
      for (int i = blockIdx.x; i < n_tiles && !*abort_flag; i += gridDim.x) {
        const int jt = i / n_mt, mt = i - jt * n_mt, row0 = jt * kGemmBN;
        const int e = segment_of(a, row0);
        const uint8_t* blob = a.pool + (int64_t)e * a.blob_stride;
        bool ok = true;
        for (int kt = 0; kt < KT; kt++) {
          const int s = issued % S;
          if (issued >= S && !mbar_wait(&empty[s], ((issued / S) - 1) & 1)) {
            set_status(a.status, kStTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          mbar_expect(&full[s], bytes);
#pragma unroll
          for (int q = 0; q < NA; q++) {
            tma_3d(tileA + (s * NA + q) * kTileBytes, &maps.a[q], kt * (kGemmBK / 2), mt * kGemmBM, e, &full[s]);
            bulk_g2s(sfA + (s * NA + q) * kSfBytes, blob + a.sfa_off[q] + ((int64_t)mt * atoms_k + APS * kt) * 512,
                     kSfBytes, &full[s]);
          }
          tma_2d(tileB + s * kTileBytes, &maps.b, kt * (kGemmBK / 2), row0, &full[s]);
          bulk_g2s(sfB + s * kSfBytes, a.sfb + ((int64_t)jt * atoms_k + APS * kt) * 512, kSfBytes, &full[s]);
          issued++;
        }
        if (!ok) break;
      }
      // No copy may still be writing this CTA's shared memory when it exits,
      // also after a timeout of any role.  A stage is reissued only after the
      // MMA consumed its previous round, so only the last S issued stages can
      // be in flight; without a timeout the MMA thread has waited for the
      // same phases, so these waits succeed at once.
      for (int n = issued > S ? issued - S : 0; n < issued; n++) mbar_wait(&full[n % S], (n / S) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer ----
      int consumed = 0, tcount = 0;
      for (int i = blockIdx.x; i < n_tiles && !*abort_flag; i += gridDim.x, tcount++) {
        const int b = tcount % NB, use = tcount / NB;
        if (use > 0 && !mbar_wait(&acc_empty[b], (use - 1) & 1)) {
          set_status(a.status, kStTimeout);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem + (uint32_t)(b * kGemmBN);  // gate/up: d0 = gate, d0 + 128 = up
        bool ok = true;
        for (int kt = 0; kt < KT; kt++) {
          const int s = consumed % S;
          if (!mbar_wait(&full[s], (consumed / S) & 1)) {
            set_status(a.status, kStTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfs = sf0 + s * SFC;
#pragma unroll
          for (int q = 0; q < NA; q++)
#pragma unroll
            for (int at = 0; at < APS; at++)
              utccp_32x128(sfs + q * 4 * APS + 4 * at, desc_sf(sfA + (s * NA + q) * kSfBytes + at * 512));
#pragma unroll
          for (int at = 0; at < APS; at++)
            utccp_32x128(sfs + 4 * APS * NA + 4 * at, desc_sf(sfB + s * kSfBytes + at * 512));
          const uint64_t bd = desc_sw128(tileB + s * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 64; kk++) {
            // MXFP4: an atom covers two MMAs of K = 64, the scale id picks
            // bytes 0-1 or 2-3 of each row's word; NVFP4: one atom an MMA
            const uint32_t byte = FMT == kFmtNv ? 0u : 2u * (kk & 1);
            const uint32_t col = FMT == kFmtNv ? 4u * kk : 4u * (kk >> 1);
#pragma unroll
            for (int q = 0; q < NA; q++) {
              const uint64_t ad = desc_sw128(tileA + (s * NA + q) * kTileBytes) + (uint64_t)(kk * 2);  // +32 B of K
              const uint32_t sa = (sfs + q * 4 * APS + col) | (byte << 30), sb = (sfs + 4 * APS * NA + col) | (byte << 30);
              if (FMT == kFmtNv)
                mma_nvf4(d0 + (uint32_t)(q * kGemmBN), ad, bd + (uint64_t)(kk * 2), idesc_nvf4(kGemmBM, kGemmBN), sa,
                         sb, (kt | kk) != 0 ? 1u : 0u);
              else
                mma_mxf4(d0 + (uint32_t)(q * kGemmBN), ad, bd + (uint64_t)(kk * 2),
                         idesc_mxf4(byte, byte, kGemmBM, kGemmBN), sa, sb, (kt | kk) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&empty[s]);
          consumed++;
        }
        if (!ok) break;
        umma_commit(&acc_full[b]);
      }
      // every tensor operation this thread issued has completed before the
      // CTA frees its tensor memory
      umma_commit(fin);
      mbar_wait(fin, 0);
    }
  } else {
    // ---- epilogue: warp w owns TMEM lanes 32(w%4).. = weight rows, and the
    // token columns [32 cg, 32 cg + 32), cg = (w - 2) / 4 ----
    const int quad = warp & 3, cg = (warp - kEpiWarp0) >> 2;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    int tcount = 0;
    for (int i = blockIdx.x; i < n_tiles; i += gridDim.x, tcount++) {
      const int b = tcount % NB, use = tcount / NB;
      if (!mbar_wait_warp(&acc_full[b], use & 1)) {
        if (lane == 0) set_status(a.status, kStTimeout);
        break;
      }
      tc_fence_after();
      const int jt = i / n_mt, mt = i - jt * n_mt, row0 = jt * kGemmBN;
      const uint32_t d0 = tmem + (uint32_t)(b * kGemmBN) + lane_off + (uint32_t)(32 * cg);
      if (MODE == 0) {
        uint32_t g0[16], g1[16], u0[16], u1[16];
        tmem_ld16_async(d0, g0);
        tmem_ld16_async(d0 + 16, g1);
        tmem_ld16_async(d0 + kGemmBN, u0);
        tmem_ld16_async(d0 + kGemmBN + 16, u1);
        tmem_wait16(g0);
        tmem_wait16(g1);
        tmem_wait16(u0);
        tmem_wait16(u1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
        const int I = a.M;
        const int irow = mt * kGemmBM + quad * 32 + lane;
        if (FMT == kFmtNv) {
          // NVFP4: g and u scaled by matrix scale x activation scale, h kept
          // in fp32 for the quantiser that follows (which needs the largest
          // |h| of the layer first); column q is padded row row0 + 32 cg + q
          const int e = segment_of(a, row0);
          const float* ts = reinterpret_cast<const float*>(a.pool + (int64_t)e * a.blob_stride + a.ts_off);
          const float sx = nv_tensor_scale(*a.amax_in).s;
          const float cgt = __fmul_rn(ts[0], sx), cut = __fmul_rn(ts[1], sx);
          float* h_col = a.hf + (size_t)(row0 + 32 * cg) * I + irow;
          // the segment's padding rows hold no token: their h is not stored
          // (the quantiser writes them as zeros)
          const int valid = (e >= a.E ? a.T : a.offs[e + 1] - a.offs[e]) - (row0 - a.pad_offs[e] + 32 * cg);
          uint32_t m = 0;
#pragma unroll
          for (int q = 0; q < 32; q++) {
            const float g = __fmul_rn(__uint_as_float(q < 16 ? g0[q & 15] : g1[q & 15]), cgt);
            const float u = __fmul_rn(__uint_as_float(q < 16 ? u0[q & 15] : u1[q & 15]), cut);
            const float hv = silu(g) * u;
            if (q < valid) {
              h_col[(size_t)q * I] = hv;
              m = max(m, __float_as_uint(hv) & 0x7fffffffu);
            }
          }
          amax_fold(m, a.amax_out);
          continue;
        }
        const int atoms_i = I / 128;
        // column q is padded row p = row0 + 32 cg + q: its codes at p * I/2 +
        // irow/2, the scale of its block 4 mt + quad at atom (jt, mt), byte
        // (p % 32) * 16 + ((p / 32) % 4) * 4 + quad = q * 16 + cg * 4 + quad
        uint8_t* hq_col = a.hq + (size_t)(row0 + 32 * cg) * (I / 2) + (irow >> 1);
        uint8_t* sf_col = a.hq_sf + ((int64_t)jt * atoms_i + mt) * 512 + cg * 4 + quad;
#pragma unroll
        for (int q = 0; q < 32; q += 2) {
          float hv[2];
#pragma unroll
          for (int e = 0; e < 2; e++) {
            const int c = q + e;
            const float g = __uint_as_float(c < 16 ? g0[c & 15] : g1[c & 15]);
            const float u = __uint_as_float(c < 16 ? u0[c & 15] : u1[c & 15]);
            hv[e] = silu(g) * u;
          }
          // the block maxima of both columns at once: the top 16 bits of |h|
          // keep its exponent field, which is all the scale rule reads
          uint32_t m = ((__float_as_uint(hv[0]) >> 16) & 0x7fffu) | (__float_as_uint(hv[1]) & 0x7fff0000u);
#pragma unroll
          for (int d = 16; d >= 1; d >>= 1) m = max_u16x2(m, __shfl_xor_sync(0xffffffffu, m, d));
#pragma unroll
          for (int e = 0; e < 2; e++) {
            const int be = (int)(((e ? m >> 16 : m) & 0x7fffu) >> 7);  // biased exponent of the block maximum
            const int e8 = min(max(be - 2, 0), 254);
            const float v = hv[e] * mx_inv_scale(e8);
            const float nb = __shfl_xor_sync(0xffffffffu, v, 1);
            if ((lane & 1) == 0) hq_col[(size_t)(q + e) * (I / 2)] = (uint8_t)cvt_e2m1x2(v, nb);
            if (lane == 0) sf_col[(q + e) * 16] = (uint8_t)e8;
          }
        }
      } else {
        uint32_t v0[16], v1[16];
        tmem_ld16_async(d0, v0);
        tmem_ld16_async(d0 + 16, v1);
        tmem_wait16(v0);
        tmem_wait16(v1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
        const int H = a.M;
        const int hrow = mt * kGemmBM + quad * 32 + lane;
        const int e = segment_of(a, row0);
        const bool shared = e >= a.E;
        const int valid = shared ? a.T : a.offs[e + 1] - a.offs[e];
        const int base_pos = shared ? a.T * a.k + (e - a.E) * a.T : a.offs[e];
        const int r0 = row0 - a.pad_offs[e] + 32 * cg;
        // NVFP4: the product of Wd's matrix scale and h's per-tensor scale
        float f = 1.f;
        if (FMT == kFmtNv)
          f = __fmul_rn(reinterpret_cast<const float*>(a.pool + (int64_t)e * a.blob_stride + a.ts_off)[2],
                        nv_tensor_scale(*a.amax_in).s);
#pragma unroll
        for (int q = 0; q < 32; q++) {
          const int r = r0 + q;
          const float v = __uint_as_float(q < 16 ? v0[q & 15] : v1[q & 15]);
          if (r < valid) a.y[(size_t)(base_pos + r) * H + hrow] = FMT == kFmtNv ? __fmul_rn(v, f) : v;
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

size_t gemm_smem_bytes(int mode, int fmt) {
  const int S = mode == 0 ? kStagesGU : kStagesDn, NA = mode == 0 ? 2 : 1, NB = mode == 0 ? 1 : 2;
  const int sf_bytes = atoms_per_stage(fmt) * 512;
  return 1024 + (size_t)S * (NA + 1) * (kTileBytes + sf_bytes) + (2 * S + 2 * NB + 1) * 8 + 16;
}

template <int MODE, int FMT>
static cudaError_t launch_one(const GemmArgs& a, const GemmMaps& maps, dim3 grid, cudaStream_t s) {
  const size_t smem = gemm_smem_bytes(MODE, FMT);
  cudaError_t e = cudaFuncSetAttribute(k_gemm<MODE, FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_gemm<MODE, FMT><<<grid, kThreads, smem, s>>>(a, maps);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmArgs& a, const GemmMaps& maps, cudaStream_t s) {
  if (a.n_tiles_max <= 0) return cudaSuccess;
  int dev = 0, nsm = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const int tiles = (a.M / kGemmBM) * a.n_tiles_max;
  const dim3 grid(tiles < nsm ? tiles : nsm);
  if (a.fmt == kFmtNv)
    return a.mode == 0 ? launch_one<0, kFmtNv>(a, maps, grid, s) : launch_one<1, kFmtNv>(a, maps, grid, s);
  return a.mode == 0 ? launch_one<0, kFmtMx>(a, maps, grid, s) : launch_one<1, kFmtMx>(a, maps, grid, s);
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

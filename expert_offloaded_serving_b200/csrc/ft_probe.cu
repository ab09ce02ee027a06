// FP4 tensor-core peak probe: the ceiling the prefill grouped GEMM is
// measured against, taken on this GPU rather than from the data sheet.
//
// One CTA per SM stages one MXFP4 operand pair in shared memory once (A: 128
// rows x 256 K, B: 128 rows x 256 K, 128-byte swizzled exactly as the GEMM's
// TMA tiles; UE8M0 scale atoms of 2^0) and copies the scales to tensor memory,
// then one thread issues `iters` rounds of four tcgen05.mma kind::mxf4 (M = N =
// 128, K = 64, the prefill GEMM's instruction) back to back into one TMEM
// accumulator, commits once and the CTA waits for the tensor pipe (bounded).
// Work = gridDim * iters * 4 * 2 * 128 * 128 * 64 FLOP; no global memory is
// read in the loop, so the time is the tensor pipe's alone.  The operands
// are a fixed non-zero code pattern (the result is not checked; the GEMM's
// parity tests check the same instruction and descriptors).
//
// Pages: prefill is the dense contraction of the method (aipolix.com,
// paragraph on bandwidth-adaptive execution); MXFP4 weights (jansverre.net,
// "Hvor raskt kjører modellene?").
#include "ft_common.cuh"
#include "ft_tc.cuh"

namespace ft {
using namespace tc;
namespace {

constexpr int kProbeThreads = 128;
constexpr int kTile = 128 * 128;  // bytes of one operand tile (128 rows x 256 e2m1)
constexpr int kCols = 256;        // TMEM columns: accumulator 128 + scale columns

__global__ void __launch_bounds__(kProbeThreads, 1) k_fp4_peak(int64_t iters, float* sink, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* A = smem;
  uint8_t* B = A + kTile;
  uint8_t* sfa = B + kTile;   // two 512-byte atoms
  uint8_t* sfb = sfa + 1024;  // two 512-byte atoms
  uint64_t* bar = reinterpret_cast<uint64_t*>(sfb + 1024);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bar + 1);
  const int warp = threadIdx.x >> 5;
  // codes: every e2m1 value appears (bytes 0x00 .. 0xff cycling), scales 2^0
  for (int i = threadIdx.x; i < 2 * kTile / 4; i += kProbeThreads)
    reinterpret_cast<uint32_t*>(A)[i] = 0x03020100u + 0x04040404u * (uint32_t)(i & 63);
  for (int i = threadIdx.x; i < 2048 / 4; i += kProbeThreads) reinterpret_cast<uint32_t*>(sfa)[i] = 0x7f7f7f7fu;
  // the tensor core reads shared memory through the async proxy
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s_u32(holder)), "r"(kCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  const uint32_t d = tmem, sf = tmem + 128;  // scales: A at +0 .. +7, B at +8 .. +15
  if (threadIdx.x == 0) {
    for (int at = 0; at < 2; at++) {
      utccp_32x128(sf + 4 * at, desc_sf(sfa + at * 512));
      utccp_32x128(sf + 8 + 4 * at, desc_sf(sfb + at * 512));
    }
    const uint64_t ad = desc_sw128(A), bd = desc_sw128(B);
    for (int64_t it = 0; it < iters; it++) {
#pragma unroll
      for (int kk = 0; kk < 4; kk++) {
        const uint32_t byte = 2u * (kk & 1), col = 4u * (kk >> 1);
        mma_mxf4(d, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc_mxf4(byte, byte, 128, 128),
                 (sf + col) | (byte << 30), (sf + 8 + col) | (byte << 30), (it | kk) != 0 ? 1u : 0u);
      }
    }
    umma_commit(bar);
  }
  __syncwarp();
  const bool done = mbar_wait_warp(bar, 0);
  if (!done && threadIdx.x == 0) set_status(status, kStTimeout);
  if (done) {
    tc_fence_after();
    float v[16];
    tmem_ld16(d + ((uint32_t)(warp * 32) << 16), v);
    // keep one value per CTA, so the accumulator is observably used
    if (threadIdx.x == 0) sink[blockIdx.x] = v[0];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols) : "memory");
  }
}

}  // namespace

size_t fp4_probe_smem() { return 1024 + 2 * kTile + 2048 + 16; }

cudaError_t launch_fp4_probe(int64_t iters, float* sink, int* status, int* grid_out, cudaStream_t s) {
  int dev = 0, nsm = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const size_t smem = fp4_probe_smem();
  if ((e = cudaFuncSetAttribute(k_fp4_peak, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
    return e;
  if (grid_out) *grid_out = nsm;
  k_fp4_peak<<<nsm, kProbeThreads, smem, s>>>(iters, sink, status);
  return cudaGetLastError();
}

}  // namespace ft

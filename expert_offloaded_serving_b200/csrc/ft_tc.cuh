// tcgen05 / TMA / mbarrier helpers (inline PTX, sm_100a) shared by the
// prefill grouped GEMM (ft_gemm.cu) and the FP4 tensor-peak probe
// (ft_probe.cu).  Descriptor bit fields follow the public PTX ISA.
#pragma once

#include <cuda.h>
#include <cstdint>
#include <cuda_runtime.h>

namespace ft {
namespace tc {

constexpr uint64_t kWaitNs = 200ull * 1000 * 1000;  // give up a wait after 200 ms

__device__ __forceinline__ uint32_t s_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(s_u32(b)), "r"(n));
}
__device__ __forceinline__ void mbar_expect(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(s_u32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint64_t gtime() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// One lane of the warp waits for phase `parity` with a short sleep between polls
// (the warps that only wait for the accumulators do not compete for issue
// slots with the producer and MMA threads), then the warp reconverges; false
// after kWaitNs of wall time.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* b, uint32_t parity) {
  uint32_t ok = 0;
  if ((threadIdx.x & 31) == 0) {
    const uint32_t a = s_u32(b);
    const uint64_t t0 = gtime();
    for (uint32_t n = 1;; n++) {
      asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                   : "=r"(ok)
                   : "r"(a), "r"(parity)
                   : "memory");
      if (ok || ((n & 15) == 0 && gtime() - t0 > kWaitNs)) break;
      __nanosleep(64);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) {  // every lane observes the completed phase (acquire) before reading its results
    uint32_t again;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                 : "=r"(again)
                 : "r"(s_u32(b)), "r"(parity)
                 : "memory");
    (void)again;
  }
  return ok != 0;
}

// wait for phase `parity`, giving up after about kWaitNs of wall time
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity) {
  const uint32_t a = s_u32(b);
  const uint64_t t0 = gtime();
  for (uint32_t n = 1;; n++) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok)
                 : "r"(a), "r"(parity)
                 : "memory");
    if (ok) return true;
    // the global timer is read on every 32nd poll only
    if ((n & 31) == 0 && gtime() - t0 > kWaitNs) return false;
  }
}

__device__ __forceinline__ void tma_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
          "r"(s_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(s_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          s_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(s_u32(bar))
      : "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   s_u32(dst)),
               "l"(src), "r"(bytes), "r"(s_u32(bar))
               : "memory");
}

// K-major, 128-byte swizzle: 8-row groups 1024 bytes apart; version 1.
__device__ __forceinline__ uint64_t desc_sw128(const void* p) {
  return (uint64_t)((s_u32(p) >> 4) & 0x3FFF) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// No swizzle, rows of 16 bytes, 8-row core matrices 128 bytes apart (scale atoms).
__device__ __forceinline__ uint64_t desc_sf(const void* p) {
  return (uint64_t)((s_u32(p) >> 4) & 0x3FFF) | (1ull << 16) | (8ull << 32) | (1ull << 46);
}

// Instruction descriptor, kind::mxf4: A, B e2m1, UE8M0 scales, K-major,
// M x N, K = 64; sf_id = byte of the scale column used.
__device__ __forceinline__ uint32_t idesc_mxf4(uint32_t a_sf_id, uint32_t b_sf_id, int M, int N) {
  return (b_sf_id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) |
         ((uint32_t)(M >> 4) << 24) | (a_sf_id << 29);
}

__device__ __forceinline__ void mma_mxf4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                         uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p; }" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
// Instruction descriptor, kind::mxf4nvf4 with UE4M3 scales (bit 23 clear),
// one per 16 elements: an MMA of K = 64 reads all four scale bytes of its
// column, so both scale ids are 0.
__device__ __forceinline__ uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_nvf4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                         uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p; }" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

__device__ __forceinline__ void utccp_32x128(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(s_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}


}  // namespace tc
}  // namespace ft

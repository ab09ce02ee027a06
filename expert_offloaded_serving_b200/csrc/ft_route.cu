// Routing kernels: fixed-order router logits, warp-per-token softmax top-k,
// and the histogram / scan / stable-scatter permutation of (token, rank) pairs.
//
// Pages: a gate picks a few experts per token and layer (aiforradalom.hu,
// "A Mixture-of-Experts (MoE) kihívásai és a FreeToken megoldásai": 6 of 256
// per layer for DeepSeek-V4-Flash).  The softmax top-k with ties to the lower
// id and the fixed summation order are this library's definitions of the step
// (see ft_moe.h).
#include "ft_common.cuh"
#include "ft_kernels.h"

namespace ft {

// ---------------------------------------------------------------------------
// router logits: warp per (expert, tile of TT tokens), fp64 accumulation
// ---------------------------------------------------------------------------
template <int TT>
__global__ void __launch_bounds__(256) k_router_logits(const uint16_t* __restrict__ x, const float* __restrict__ wr,
                                                       int T, int H, int E, float* __restrict__ logits) {
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.y * 8 + (threadIdx.x >> 5);
  const int t0 = blockIdx.x * TT;
  if (e >= E) return;
  double acc[TT];
#pragma unroll
  for (int i = 0; i < TT; i++) acc[i] = 0.0;
  const float4* wrow = reinterpret_cast<const float4*>(wr + (size_t)e * H);
  const int C = H >> 7;  // 128 elements per step: 4 consecutive per lane
  for (int c = 0; c < C; c++) {
    float4 w4 = __ldg(wrow + c * 32 + lane);
#pragma unroll
    for (int i = 0; i < TT; i++) {
      if (t0 + i < T) {
        uint2 xv = __ldg(reinterpret_cast<const uint2*>(x + (size_t)(t0 + i) * H + c * 128 + lane * 4));
        double a = acc[i];
        // ascending k inside the lane; products bf16*fp32 are exact in fp64
        a += (double)bf16_bits_to_f32((uint16_t)(xv.x & 0xffff)) * (double)w4.x;
        a += (double)bf16_bits_to_f32((uint16_t)(xv.x >> 16)) * (double)w4.y;
        a += (double)bf16_bits_to_f32((uint16_t)(xv.y & 0xffff)) * (double)w4.z;
        a += (double)bf16_bits_to_f32((uint16_t)(xv.y >> 16)) * (double)w4.w;
        acc[i] = a;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < TT; i++) {
    double a = acc[i];
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) a = a + __shfl_xor_sync(0xffffffffu, a, d);
    if (lane == 0 && t0 + i < T) logits[(size_t)(t0 + i) * E + e] = __double2float_rn(a);
  }
}

// ---------------------------------------------------------------------------
// router logits for many tokens: the same summation order, register-tiled.
// A CTA of 8 warps takes 32 tokens x 16 experts; warp w takes tokens
// 8(w/2) .. +7 and experts 8(w%2) .. +7, and lane j holds partial sum j of
// each of its warp's 64 (token, expert) pairs in registers.  Per 128-element
// block of K the CTA stages x and Wr in shared memory as fp64 (each value
// converted once), element 4j + v of the block at [v][j] so that lane j's
// reads are consecutive; the global loads run two blocks ahead.  Lane j adds
// its block elements 4j, 4j+1, 4j+2, 4j+3 in ascending order, so every
// partial sum sees the same terms in the same order as in k_router_logits;
// the butterfly and the rounding are the same.
// ---------------------------------------------------------------------------
constexpr int kRtT = 32, kRtE = 16;
constexpr size_t kRtSmem = 2 * (size_t)(kRtT + kRtE) * 128 * 8;

// fp32 -> fp64, exact: normal values by moving the fields (rebiased
// exponent, mantissa widened), zeros, subnormals, infinities and NaNs by the
// conversion instruction.
__device__ __forceinline__ double f32_to_f64(float f) {
  const uint32_t u = __float_as_uint(f), e = (u >> 23) & 0xffu;
  if (e == 0u || e == 255u) return (double)f;
  const uint32_t hi = (u & 0x80000000u) | ((e + 896u) << 20) | ((u >> 3) & 0xfffffu);
  return __hiloint2double((int)hi, (int)(u << 29));
}

__global__ void __launch_bounds__(256, 1) k_router_logits_tiled(const uint16_t* __restrict__ x,
                                                                const float* __restrict__ wr, int T, int H, int E,
                                                                float* __restrict__ logits) {
  extern __shared__ __align__(16) uint8_t rt_smem[];
  double* xs = reinterpret_cast<double*>(rt_smem);  // [2][kRtT][4][32]
  double* ws = xs + 2 * kRtT * 128;                 // [2][kRtE][4][32]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tw = warp >> 1, ew = warp & 1;
  const int t0 = blockIdx.x * kRtT, e0 = blockIdx.y * kRtE;
  // staging: lane j of warp w loads elements 4j .. 4j+3 of tokens w, w + 8,
  // w + 16, w + 24 and of experts w, w + 8, and stores element 4j + v at
  // [v][j]: a warp's loads are contiguous and its stores 32 consecutive
  // doubles (no bank conflicts)
  const uint2* xg[4];
  bool tok_ok[4];
#pragma unroll
  for (int m = 0; m < 4; m++) {
    const int t = t0 + warp + 8 * m;
    tok_ok[m] = t < T;
    xg[m] = reinterpret_cast<const uint2*>(x + (size_t)(tok_ok[m] ? t : 0) * H) + lane;
  }
  const float4* wg[2];
  bool exp_ok[2];
#pragma unroll
  for (int m = 0; m < 2; m++) {
    const int e = e0 + warp + 8 * m;
    exp_ok[m] = e < E;
    wg[m] = reinterpret_cast<const float4*>(wr + (size_t)(exp_ok[m] ? e : 0) * H) + lane;
  }
  // two register sets of staged loads, named apart so that a set chosen at
  // run time still lives in registers
  uint2 xr0[4], xr1[4];
  float4 wq0[2], wq1[2];
  auto gload_into = [&](int c, uint2 (&xr)[4], float4 (&wq)[2]) {
#pragma unroll
    for (int m = 0; m < 4; m++) xr[m] = tok_ok[m] ? __ldg(xg[m] + c * 32) : make_uint2(0u, 0u);
#pragma unroll
    for (int m = 0; m < 2; m++) wq[m] = exp_ok[m] ? __ldg(wg[m] + c * 32) : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  auto gload = [&](int c, int set) {
    if (set == 0) gload_into(c, xr0, wq0);
    else gload_into(c, xr1, wq1);
  };
  auto sstore_from = [&](int buf, const uint2 (&xr)[4], const float4 (&wq)[2]) {
#pragma unroll
    for (int m = 0; m < 4; m++) {
      double* xd = xs + ((size_t)buf * kRtT + warp + 8 * m) * 128 + lane;
      xd[0] = f32_to_f64(bf16_bits_to_f32((uint16_t)(xr[m].x & 0xffffu)));
      xd[32] = f32_to_f64(bf16_bits_to_f32((uint16_t)(xr[m].x >> 16)));
      xd[64] = f32_to_f64(bf16_bits_to_f32((uint16_t)(xr[m].y & 0xffffu)));
      xd[96] = f32_to_f64(bf16_bits_to_f32((uint16_t)(xr[m].y >> 16)));
    }
#pragma unroll
    for (int m = 0; m < 2; m++) {
      double* wd = ws + ((size_t)buf * kRtE + warp + 8 * m) * 128 + lane;
      wd[0] = f32_to_f64(wq[m].x);
      wd[32] = f32_to_f64(wq[m].y);
      wd[64] = f32_to_f64(wq[m].z);
      wd[96] = f32_to_f64(wq[m].w);
    }
  };
  auto sstore = [&](int buf, int set) {
    if (set == 0) sstore_from(buf, xr0, wq0);
    else sstore_from(buf, xr1, wq1);
  };
  double acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; i++)
#pragma unroll
    for (int j = 0; j < 8; j++) acc[i][j] = 0.0;
  const int C = H >> 7;
  // register set s holds the global loads of block c with c & 1 == s; block
  // c + 1 is stored while block c is used, block c + 3 loaded
  gload(0, 0);
  if (C > 1) gload(1, 1);
  sstore(0, 0);
  if (C > 2) gload(2, 0);
  __syncthreads();
  for (int c = 0; c < C; c++) {
    const int buf = c & 1;
    const double* xb = xs + ((size_t)buf * kRtT + 8 * tw) * 128 + lane;
    const double* wb = ws + ((size_t)buf * kRtE + 8 * ew) * 128 + lane;
#pragma unroll
    for (int v = 0; v < 4; v++) {
      double xv[8], wv[8];
#pragma unroll
      for (int i = 0; i < 8; i++) xv[i] = xb[i * 128 + v * 32];
#pragma unroll
      for (int j = 0; j < 8; j++) wv[j] = wb[j * 128 + v * 32];
      // products bf16 * fp32 are exact in fp64: fma == add of the product
#pragma unroll
      for (int i = 0; i < 8; i++)
#pragma unroll
        for (int j = 0; j < 8; j++) acc[i][j] = fma(xv[i], wv[j], acc[i][j]);
    }
    if (c + 1 < C) sstore(buf ^ 1, (c + 1) & 1);
    if (c + 3 < C) gload(c + 3, (c + 1) & 1);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; i++)
#pragma unroll
    for (int j = 0; j < 8; j++) {
      double a = acc[i][j];
#pragma unroll
      for (int d = 16; d >= 1; d >>= 1) a = a + __shfl_xor_sync(0xffffffffu, a, d);
      const int t = t0 + 8 * tw + i, e = e0 + 8 * ew + j;
      if (lane == ((i * 8 + j) & 31) && t < T && e < E) logits[(size_t)t * E + e] = __double2float_rn(a);
    }
}

cudaError_t launch_router_logits(const uint16_t* x, const float* wr, int T, int H, int E, float* logits,
                                 cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  dim3 block(256);
  if (T <= 4) {
    dim3 grid((T + 3) / 4, (E + 7) / 8);
    k_router_logits<4><<<grid, block, 0, s>>>(x, wr, T, H, E, logits);
  } else if (T < 64) {
    dim3 grid((T + 7) / 8, (E + 7) / 8);
    k_router_logits<8><<<grid, block, 0, s>>>(x, wr, T, H, E, logits);
  } else {
    dim3 grid((T + kRtT - 1) / kRtT, (E + kRtE - 1) / kRtE);
    cudaError_t e = cudaFuncSetAttribute(k_router_logits_tiled, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kRtSmem);
    if (e != cudaSuccess) return e;
    k_router_logits_tiled<<<grid, block, kRtSmem, s>>>(x, wr, T, H, E, logits);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// softmax top-k: one warp per token
// ---------------------------------------------------------------------------
struct Cand {
  float v;
  int i;  // -1 = none
};

// a ranks before b: valid first, non-NaN first, larger value, lower id
__device__ __forceinline__ bool better(const Cand& a, const Cand& b) {
  if (a.i < 0) return false;
  if (b.i < 0) return true;
  bool an = isnan(a.v), bn = isnan(b.v);
  if (an != bn) return !an;
  if (!an && a.v != b.v) return a.v > b.v;
  return a.i < b.i;
}

constexpr int kMaxE = 1024;
constexpr int kMaxK = 16;

__global__ void __launch_bounds__(256) k_topk(const float* __restrict__ logits, int T, int E, int k, int renorm,
                                              int32_t* __restrict__ ids, float* __restrict__ w, int* status) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* row = logits + (size_t)t * E;
  float v[kMaxE / 32];
  uint32_t taken = 0;
  const int per = (E + 31) >> 5;
  bool bad = false;
  float vmax = -INFINITY;
#pragma unroll
  for (int q = 0; q < kMaxE / 32; q++) {
    if (q < per) {
      int e = lane + 32 * q;
      float x = e < E ? row[e] : -INFINITY;
      v[q] = x;
      if (e < E) {
        if (isnan(x) || x == INFINITY) bad = true;
        if (!isnan(x)) vmax = fmaxf(vmax, x);
      }
    }
  }
  // a row with no finite logit is also invalid
  for (int d = 16; d >= 1; d >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, d));
  if (vmax == -INFINITY) bad = true;
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(status, kStNonfinite);

  float sel_v[kMaxK];
  int sel_i[kMaxK];
#pragma unroll
  for (int r = 0; r < kMaxK; r++) {
    if (r < k) {
      Cand best{0.f, -1};
#pragma unroll
      for (int q = 0; q < kMaxE / 32; q++) {
        int e = lane + 32 * q;
        if (q < per && e < E && !((taken >> q) & 1u)) {
          Cand c{v[q], e};
          if (better(c, best)) best = c;
        }
      }
#pragma unroll
      for (int d = 16; d >= 1; d >>= 1) {
        Cand o{__shfl_xor_sync(0xffffffffu, best.v, d), __shfl_xor_sync(0xffffffffu, best.i, d)};
        if (better(o, best)) best = o;
      }
      sel_v[r] = best.v;
      sel_i[r] = best.i;
      if (best.i >= 0 && (best.i & 31) == lane) taken |= 1u << (best.i >> 5);
    }
  }
  // weights
  const float m = sel_v[0];
  float denom = 0.f;
  if (renorm) {
#pragma unroll
    for (int r = 0; r < kMaxK; r++)
      if (r < k) denom += expf(sel_v[r] - m);
  } else {
    float part = 0.f;
#pragma unroll
    for (int q = 0; q < kMaxE / 32; q++) {
      int e = lane + 32 * q;
      if (q < per && e < E) part += expf(v[q] - m);
    }
    for (int d = 16; d >= 1; d >>= 1) part += __shfl_xor_sync(0xffffffffu, part, d);
    denom = part;
  }
#pragma unroll
  for (int r = 0; r < kMaxK; r++) {
    if (r < k && lane == r) {
      ids[(size_t)t * k + r] = sel_i[r];
      w[(size_t)t * k + r] = expf(sel_v[r] - m) / denom;
    }
  }
}

cudaError_t launch_topk(const float* logits, int T, int E, int k, int renorm, int32_t* ids, float* w, int* status,
                        cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  k_topk<<<(T + 7) / 8, 256, 0, s>>>(logits, T, E, k, renorm, ids, w, status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// permutation: one CTA of 32 warps; warp w owns a contiguous range of pairs.
//   phase 1  per-warp histograms cnt[w][e] (match_any groups inside a warp)
//   phase 2  per-expert exclusive prefix over warps, scan over experts
//   phase 3  stable scatter: pos = offs[e] + before-this-warp + rank in warp
// Also writes the ascending list of experts with at least one pair and, when
// pad_offs != NULL, segment starts padded to multiples of 128 rows.
// ---------------------------------------------------------------------------
constexpr int kPermWarps = 32;

__device__ __forceinline__ int block_excl_scan(int v, int* warp_tot, int* total) {
  // 1024 threads; returns the exclusive prefix of v in thread order
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, d);
    if (lane >= d) x += y;
  }
  if (lane == 31) warp_tot[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int t = warp_tot[lane];
    int xs = t;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, xs, d);
      if (lane >= d) xs += y;
    }
    warp_tot[lane] = xs - t;
    if (lane == 31) *total = xs;
  }
  __syncthreads();
  int r = warp_tot[wid] + x - v;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(1024) k_permute(const int32_t* __restrict__ ids, int P, int E,
                                                  int32_t* __restrict__ offs, int32_t* __restrict__ perm,
                                                  int32_t* __restrict__ inv, int32_t* __restrict__ active,
                                                  int32_t* __restrict__ n_active, int32_t* __restrict__ pad_offs,
                                                  int* status) {
  extern __shared__ int smem[];
  int* cnt = smem;                          // [32][E]
  int* offs_s = cnt + kPermWarps * E;       // [E]
  __shared__ int warp_tot[32];
  __shared__ int total;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kPermWarps * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const int chunk = ((P + kPermWarps * 32 - 1) / (kPermWarps * 32)) * 32;
  const int beg = wid * chunk, end = min(P, beg + chunk);
  const unsigned lt = (1u << lane) - 1u;
  for (int g = beg; g < end; g += 32) {
    int f = g + lane;
    int e = f < end ? ids[f] : -1;
    if (f < end && (e < 0 || e >= E)) {
      set_status(status, kStBadId);
      e = -1;
    }
    unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lt) == 0) cnt[wid * E + e] += __popc(peers);
  }
  __syncthreads();
  // phase 2 (E <= 1024, one expert per thread): exclusive prefix over warps,
  // then scans over experts for offsets, the active list and padded offsets
  {
    const int e = threadIdx.x;
    int tot = 0;
    if (e < E) {
      for (int w2 = 0; w2 < kPermWarps; w2++) {
        int c = cnt[w2 * E + e];
        cnt[w2 * E + e] = tot;
        tot += c;
      }
    }
    int ex = block_excl_scan(tot, warp_tot, &total);
    if (e < E) {
      offs[e] = ex;
      offs_s[e] = ex;
    }
    if (threadIdx.x == 0) offs[E] = total;
    int flag = (e < E && tot > 0) ? 1 : 0;
    int pos = block_excl_scan(flag, warp_tot, &total);
    if (flag) active[pos] = e;
    if (threadIdx.x == 0) *n_active = total;
    if (pad_offs != nullptr) {
      int pp = block_excl_scan(e < E ? (int)pad_up(tot, 128) : 0, warp_tot, &total);
      if (e < E) pad_offs[e] = pp;
      if (threadIdx.x == 0) pad_offs[E] = total;
    }
    __syncthreads();
  }
  // phase 3: stable scatter
  for (int g = beg; g < end; g += 32) {
    int f = g + lane;
    int e = f < end ? ids[f] : -1;
    if (e >= E) e = -1;
    unsigned peers = __match_any_sync(0xffffffffu, e);
    int before = 0;
    if (e >= 0) before = cnt[wid * E + e];
    __syncwarp();
    if (e >= 0) {
      int pos = offs_s[e] + before + __popc(peers & lt);
      perm[pos] = f;
      inv[f] = pos;
      if ((peers & lt) == 0) cnt[wid * E + e] = before + __popc(peers);
    }
    __syncwarp();
  }
}

size_t permute_smem_bytes(int E) { return (size_t)(kPermWarps * E + E) * sizeof(int); }

cudaError_t launch_permute(const int32_t* ids, int P, int E, int32_t* offs, int32_t* perm, int32_t* inv,
                           int32_t* active, int32_t* n_active, int32_t* pad_offs, int* status, cudaStream_t s) {
  size_t sm = permute_smem_bytes(E);
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(k_permute, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    attr_set = true;
  }
  k_permute<<<1, 1024, sm, s>>>(ids, P, E, offs, perm, inv, active, n_active, pad_offs, status);
  return cudaGetLastError();
}

}  // namespace ft

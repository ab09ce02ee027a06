// Decode path for small batches (T <= 16).
//
//   k_route         one CTA per layer: softmax top-k of the T tokens and the
//                   permutation of their (token, rank) pairs by expert, stored
//                   as a compact routing record (distinct experts = units).
//   k_dec_gate_up   CTA = (unit, block of R rows of Wg and Wu) over the full K:
//                   the tile is staged in shared memory with coalesced 16-byte
//                   cp.async copies; tpr threads share a row, each dequantising
//                   its scale-atom columns of e2m1 codes with their UE8M0 scales
//                   in registers (split-K inside the row group, reduced by
//                   shuffles); gate and up share the activation reads; SwiGLU
//                   gives fp32 h.
//   k_dec_down      CTA = (unit, block of R rows of Wd) over K = I; launched as a
//                   programmatic dependent of gate/up, so its tile streams in
//                   while gate/up runs; after griddepcontrol.wait it reads h and
//                   writes y.  The last CTA to finish a row block (an atomic
//                   counter per block) sums w[t][j] * y over j ascending plus
//                   the shared expert and rounds once to bf16.
//
// Pages: decode fetches or reuses the selected experts and sums their partial
// results exactly (jansverre.net, "Hvorfor er båndbredden viktigere enn antall
// kjerner?"); a gate picks a few experts per token (aiforradalom.hu, "A
// Mixture-of-Experts (MoE) kihívásai és a FreeToken megoldásai").
#include "ft_common.cuh"
#include "ft_decode.h"

namespace ft {
namespace {

constexpr int kThreads = 256;       // routing kernel
constexpr int kGemvThreads = 512;   // GEMV kernels
constexpr int kRows = 128;        // rows per CTA tile (one scale-atom row block)

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }


// ---------------------------------------------------------------------------
// routing inside a CTA
// ---------------------------------------------------------------------------
// Per-CTA shared header of the GEMV kernels, then the tiles.
struct CtaHdr {
  int32_t tok[16];
  int32_t last;
  int32_t pad[3];
};
constexpr size_t kTileOff = 128;

// Order key of a logit: larger key = ranks first.  NaN -> 1 (below -inf),
// -0 -> +0, absent -> 0.
__device__ __forceinline__ uint32_t order_key(float v) {
  uint32_t b = __float_as_uint(v);
  if (isnan(v)) return 1u;
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Warp w routes tokens w, w+8, ...; then every thread finds the permuted
// position of its pair; finally units (distinct experts, ascending) are listed.
// PER = logits per lane (E <= 32 * PER), a compile-time bound so that the keys
// stay in registers.
template <int PER>
__device__ void route_in_cta(const float* __restrict__ logits, int T, int E, int k, int renorm, Route& r,
                             int* status) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) r.bad = 0;
  __syncthreads();
  for (int t = warp; t < T; t += kThreads / 32) {
    const float* row = logits + (size_t)t * E;
    uint32_t key[PER];
    bool bad = false;
    float vmax = -INFINITY;
#pragma unroll
    for (int q = 0; q < PER; q++) {
      int e = lane + 32 * q;
      float v = e < E ? __ldg(row + e) : -INFINITY;
      key[q] = e < E ? order_key(v) : 0u;
      if (e < E && (isnan(v) || v == INFINITY)) bad = true;
      if (e < E && !isnan(v)) vmax = fmaxf(vmax, v);
    }
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 16));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 8));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 4));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 2));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 1));
    if (vmax == -INFINITY) bad = true;
    if (__any_sync(0xffffffffu, bad) && lane == 0) r.bad = 1;
    float my_v = 0.f;
    int my_id = -1;
    for (int j = 0; j < k; j++) {
      // lane-local best: largest key, lowest id (ids ascend with q)
      uint32_t bk = key[0];
      int bq = 0;
#pragma unroll
      for (int q = 1; q < PER; q++)
        if (key[q] > bk) {
          bk = key[q];
          bq = q;
        }
      const uint32_t kmax = __reduce_max_sync(0xffffffffu, bk);
      const uint32_t cand = (bk == kmax && bk != 0u) ? (uint32_t)(lane + 32 * bq) : 0xffffffffu;
      const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
      if ((int)(win & 31) == lane) {
#pragma unroll
        for (int q = 0; q < PER; q++)
          if (q == bq) key[q] = 0u;
      }
      if (lane == j) {
        my_id = (int)win;
        my_v = win < (uint32_t)E ? __ldg(row + win) : -INFINITY;
      }
    }
    // weights: softmax at the chosen ids (renormalised over k, or over all E)
    float m = __shfl_sync(0xffffffffu, my_v, 0);
    float ex = (lane < k) ? expf(my_v - m) : 0.f;
    float denom;
    if (renorm) {
      denom = ex;
      for (int d = 16; d >= 1; d >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, d);
    } else {
      float part = 0.f;
#pragma unroll
      for (int q = 0; q < PER; q++) {
        int e = lane + 32 * q;
        if (e < E) part += expf(__ldg(row + e) - m);
      }
      for (int d = 16; d >= 1; d >>= 1) part += __shfl_xor_sync(0xffffffffu, part, d);
      denom = part;
    }
    if (lane < k) {
      r.ids[t * k + lane] = my_id;
      r.w[t * k + lane] = ex / denom;
    }
  }
  __syncthreads();
  const int P = T * k;
  // permuted position of pair f: pairs of lower experts, then same expert at
  // lower tokens; `first` marks the lowest-token pair of each expert
  for (int f = threadIdx.x; f < P; f += kThreads) {
    int e = r.ids[f], t = f / k;
    int pos = 0;
    bool first = true;
    for (int f2 = 0; f2 < P; f2++) {
      int e2 = r.ids[f2], t2 = f2 / k;
      pos += (e2 < e) || (e2 == e && t2 < t);
      if (e2 == e && t2 < t) first = false;
    }
    r.pos[f] = pos;
    r.perm[pos] = f;
    r.first[f] = first ? 1 : 0;
  }
  __syncthreads();
  // units = distinct experts in ascending order
  for (int f = threadIdx.x; f < P; f += kThreads) {
    if (!r.first[f]) continue;
    int e = r.ids[f];
    int unit = 0, cnt = 0;
    for (int f2 = 0; f2 < P; f2++) {
      int e2 = r.ids[f2];
      unit += (r.first[f2] && e2 < e);
      cnt += (e2 == e);
    }
    r.unit_e[unit] = e;
    r.unit_p0[unit] = r.pos[f];
    r.unit_m[unit] = cnt;
  }
  if (threadIdx.x == 0) {
    int n = 0;
    for (int f = 0; f < P; f++) n += r.first[f];
    r.n_active = n;
    if (r.bad) set_status(status, kStNonfinite);
  }
  __syncthreads();
}

struct UnitInfo {
  int e, m, hbase;
  bool shared;
};

// Unit u of the layer's routing record: a distinct selected expert (ascending
// id) or, past max_units, a shared expert.  Token ids of the unit go to tok[].
__device__ __forceinline__ bool resolve_unit(const DecodeArgs& a, const Route* __restrict__ rec, int u, UnitInfo& ui,
                                             int* tok) {
  if (u < a.max_units) {
    if (u >= rec->n_active) return false;
    ui.e = rec->unit_e[u];
    ui.m = rec->unit_m[u];
    ui.hbase = rec->unit_p0[u];
    ui.shared = false;
  } else {
    int s = u - a.max_units;
    ui.e = a.E + s;
    ui.m = a.T;
    ui.hbase = a.T * a.k + s * a.T;
    ui.shared = true;
  }
  if (threadIdx.x < ui.m) tok[threadIdx.x] = ui.shared ? threadIdx.x : rec->perm[ui.hbase + threadIdx.x] / a.k;
  return true;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Dot of 32 e2m1 codes (16 bytes) with 32 activations read as 8 float4 from
// shared memory at `x` with a stride of `xs` float4 between consecutive ones.
__device__ __forceinline__ float chunk_dot(uint4 q, const float4* x, int xs) {
  float2 p0 = make_float2(0.f, 0.f), p1 = make_float2(0.f, 0.f);
  const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int wv = 0; wv < 4; wv++) {
    const float4 xa = x[(2 * wv) * xs], xb = x[(2 * wv + 1) * xs];
    p0 = ffma2(f16x2_to_f32x2(e2m1x2_to_f16x2(qs[wv])), make_float2(xa.x, xa.y), p0);
    p1 = ffma2(f16x2_to_f32x2(e2m1x2_to_f16x2(qs[wv] >> 8)), make_float2(xa.z, xa.w), p1);
    p0 = ffma2(f16x2_to_f32x2(e2m1x2_to_f16x2(qs[wv] >> 16)), make_float2(xb.x, xb.y), p0);
    p1 = ffma2(f16x2_to_f32x2(e2m1x2_to_f16x2(qs[wv] >> 24)), make_float2(xb.z, xb.w), p1);
  }
  return (p0.x + p0.y) + (p1.x + p1.y);
}

// ---------------------------------------------------------------------------
// CTA geometry (host and device).  A CTA takes R consecutive weight rows over
// the full K of one unit.  tpr threads share a row: thread `sub` owns apr
// scale-atom columns (128 elements each) sub*apr .. sub*apr+apr-1.  Shared
// memory holds the R rows' codes, their scale words and the activations of
// MT tokens, each laid out so that the tpr threads of a row read consecutive
// 16-byte words (no bank conflicts):
//   codes: row r, logical chunk c = 4*atom + j, atom = sub*apr + al  ->
//          16-byte slot r*chunks + (al*4 + j)*tpr + sub
//   acts:  token t, float4 f = atom*32 + j*8 + v  ->  t*K/4 + ((al*4 + j)*8 + v)*tpr + sub
//   scales: row r, atom -> word r*atoms + atom (4 blocks' bytes)
// ---------------------------------------------------------------------------
constexpr int kMT = 2;            // tokens per pass over the tile
constexpr size_t kSmemLimit = 220 * 1024;

struct Geo {
  int K, atoms, tpr, apr, R, threads, nmat;
  size_t codes, scales, act, total;
};

__host__ __device__ inline Geo make_geo(int K, int rows, int nmat) {
  Geo g;
  g.K = K;
  g.nmat = nmat;
  g.atoms = K / 128;
  g.tpr = 16;
  while (g.tpr > 1 && g.atoms % g.tpr) g.tpr >>= 1;
  g.apr = g.atoms / g.tpr;
  g.R = kGemvThreads / g.tpr;
  if (g.R > 128) g.R = 128;
  if (g.R > rows) g.R = rows;
  for (;;) {
    g.codes = kTileOff;
    g.scales = g.codes + (size_t)nmat * g.R * K / 2;
    g.act = g.scales + (size_t)nmat * g.R * g.atoms * 4;
    g.total = g.act + (size_t)kMT * K * 4;
    if (g.total <= kSmemLimit || g.R <= 8) break;
    g.R >>= 1;
  }
  g.threads = g.R * g.tpr;
  return g;
}

// Stage rows [row0, row0 + R) of one matrix (codes at `codes_g`, row pitch
// K/2; scale region `sc_g`) with cp.async.
__device__ __forceinline__ void stage_rows(const Geo& g, uint8_t* codes_s, uint32_t* sc_s, const uint8_t* codes_g,
                                           const uint8_t* sc_g, int row0) {
  const int chunks = g.K / 32;
  const uint8_t* src = codes_g + (size_t)row0 * (g.K / 2);
  for (int i = threadIdx.x; i < g.R * chunks; i += g.threads) {
    const int r = i / chunks, c = i - r * chunks;
    const int atom = c >> 2, j = c & 3, sub = atom / g.apr, al = atom - sub * g.apr;
    cp_async16(codes_s + ((size_t)r * chunks + (al * 4 + j) * g.tpr + sub) * 16, src + (size_t)i * 16);
  }
  for (int i = threadIdx.x; i < g.R * g.atoms; i += g.threads) {
    const int r = i / g.atoms, atom = i - r * g.atoms;
    cp_async4(sc_s + i, sc_g + sf_word(row0 + r, atom, g.atoms));
  }
}

// Stage tokens tok[t0 .. t0+n) of x (bf16 [.][K]) or of h (fp32 rows) as fp32
// in the swizzled activation layout.
template <bool BF16>
__device__ __forceinline__ void stage_act(const Geo& g, float* act, const void* src, const int* rowidx, int n) {
  const int f4 = g.K / 4;
  for (int i = threadIdx.x; i < kMT * f4; i += g.threads) {
    const int t = i / f4, f = i - t * f4;
    const int atom = f >> 5, jv = f & 31, sub = atom / g.apr, al = atom - sub * g.apr;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < n) {
      if (BF16) {
        const uint2 w = *reinterpret_cast<const uint2*>((const uint16_t*)src + (size_t)rowidx[t] * g.K + f * 4);
        v = make_float4(bf16_bits_to_f32(w.x & 0xffff), bf16_bits_to_f32(w.x >> 16), bf16_bits_to_f32(w.y & 0xffff),
                        bf16_bits_to_f32(w.y >> 16));
      } else {
        v = *reinterpret_cast<const float4*>((const float*)src + (size_t)rowidx[t] * g.K + f * 4);
      }
    }
    reinterpret_cast<float4*>(act)[(size_t)t * f4 + ((al * 32 + jv) * g.tpr + sub)] = v;
  }
}

// Row-partial dots of this thread's atoms for matrix `mat` and the (up to)
// kMT staged tokens; reduced over the tpr threads of the row.
__device__ __forceinline__ void row_dots(const Geo& g, const uint8_t* codes_s, const uint32_t* sc_s, const float* act,
                                         int mat, int r, int sub, int n, float* out) {
  const int chunks = g.K / 32;
  const int f4 = g.K / 4;
  const uint8_t* cs = codes_s + (size_t)mat * g.R * g.K / 2 + (size_t)r * chunks * 16;
  const uint32_t* ss = sc_s + (size_t)mat * g.R * g.atoms + (size_t)r * g.atoms;
  float s0 = 0.f, s1 = 0.f;
  for (int al = 0; al < g.apr; al++) {
    const uint32_t sw = ss[sub * g.apr + al];
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const uint4 q = *reinterpret_cast<const uint4*>(cs + ((al * 4 + j) * g.tpr + sub) * 16);
      const float sc = ue8m0_to_f32((sw >> (8 * j)) & 0xff);
      const float4* x0 = reinterpret_cast<const float4*>(act) + ((al * 4 + j) * 8) * g.tpr + sub;
      s0 = fmaf(chunk_dot(q, x0, g.tpr), sc, s0);
      if (n > 1) s1 = fmaf(chunk_dot(q, x0 + f4, g.tpr), sc, s1);
    }
  }
  for (int d = g.tpr >> 1; d >= 1; d >>= 1) {
    s0 += __shfl_xor_sync(0xffffffffu, s0, d);
    s1 += __shfl_xor_sync(0xffffffffu, s1, d);
  }
  out[0] = s0;
  out[1] = s1;
}

}  // namespace

// ---------------------------------------------------------------------------
// gate/up + SwiGLU: CTA = (unit, block of R rows of Wg and Wu), full K = H
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kGemvThreads) k_dec_gate_up(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  CtaHdr& hd = *reinterpret_cast<CtaHdr*>(smem);
  const Geo g = make_geo(a.H, a.I, 2);
  uint8_t* codes_s = smem + g.codes;
  uint32_t* sc_s = reinterpret_cast<uint32_t*>(smem + g.scales);
  float* act = reinterpret_cast<float*>(smem + g.act);
  const int nrb = a.I / g.R;
  const int rb = blockIdx.x % nrb, u = blockIdx.x / nrb;
  UnitInfo ui;
  if (!resolve_unit(a, a.rec, u, ui, hd.tok)) {
    pdl_trigger();
    return;
  }
  const uint8_t* blob = a.eptr[ui.e];
  if (blob == nullptr) {
    if (threadIdx.x == 0) set_status(a.status, kStMissing);
    pdl_trigger();
    return;
  }
  const int row0 = rb * g.R;
  stage_rows(g, codes_s, sc_s, blob + a.lay.wg, blob + a.lay.wg_sf, row0);
  stage_rows(g, codes_s + (size_t)g.R * a.H / 2, sc_s + (size_t)g.R * g.atoms, blob + a.lay.wu, blob + a.lay.wu_sf,
             row0);
  cp_async_commit();
  pdl_trigger();
  pdl_wait();  // x is the previous kernel's output when launched as a dependent
  const int r = threadIdx.x / g.tpr, sub = threadIdx.x % g.tpr;
  for (int t0 = 0; t0 < ui.m; t0 += kMT) {
    const int n = min(kMT, ui.m - t0);
    __syncthreads();
    stage_act<true>(g, act, a.x, hd.tok + t0, n);
    cp_async_wait_all();
    __syncthreads();
    float gs[2], us[2];
    row_dots(g, codes_s, sc_s, act, 0, r, sub, n, gs);
    row_dots(g, codes_s, sc_s, act, 1, r, sub, n, us);
    if (sub == 0) {
      a.h[(size_t)(ui.hbase + t0) * a.I + row0 + r] = silu(gs[0]) * us[0];
      if (n > 1) a.h[(size_t)(ui.hbase + t0 + 1) * a.I + row0 + r] = silu(gs[1]) * us[1];
    }
  }
}

// ---------------------------------------------------------------------------
// down + combine: CTA = (unit, block of R rows of Wd), full K = I.  The last
// CTA to finish a row block (one counter per block) does the weighted combine.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kGemvThreads) k_dec_down(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  CtaHdr& hd = *reinterpret_cast<CtaHdr*>(smem);
  const Geo g = make_geo(a.I, a.H, 1);
  uint8_t* codes_s = smem + g.codes;
  uint32_t* sc_s = reinterpret_cast<uint32_t*>(smem + g.scales);
  float* act = reinterpret_cast<float*>(smem + g.act);
  const int nrb = a.H / g.R;
  const int rb = blockIdx.x % nrb, u = blockIdx.x / nrb;
  UnitInfo ui;
  if (!resolve_unit(a, a.rec, u, ui, hd.tok)) {
    pdl_trigger();
    return;
  }
  const uint8_t* blob = a.eptr[ui.e];
  if (blob == nullptr) {
    pdl_trigger();
    return;  // already reported by the gate/up kernel
  }
  const int row0 = rb * g.R;
  stage_rows(g, codes_s, sc_s, blob + a.lay.wd, blob + a.lay.wd_sf, row0);
  cp_async_commit();
  pdl_trigger();
  pdl_wait();  // h is written by the gate/up kernel
  if (threadIdx.x < 16) hd.tok[threadIdx.x] = ui.hbase + threadIdx.x;  // h rows of the unit's tokens
  const int r = threadIdx.x / g.tpr, sub = threadIdx.x % g.tpr;
  for (int t0 = 0; t0 < ui.m; t0 += kMT) {
    const int n = min(kMT, ui.m - t0);
    __syncthreads();
    stage_act<false>(g, act, a.h, hd.tok + t0, n);
    cp_async_wait_all();
    __syncthreads();
    float ys[2];
    row_dots(g, codes_s, sc_s, act, 0, r, sub, n, ys);
    if (sub == 0) {
      a.y[(size_t)(ui.hbase + t0) * a.H + row0 + r] = ys[0];
      if (n > 1) a.y[(size_t)(ui.hbase + t0 + 1) * a.H + row0 + r] = ys[1];
    }
  }
  // last CTA of this row block combines
  __threadfence();
  __syncthreads();
  const int units = a.rec->n_active + a.n_shared;
  if (threadIdx.x == 0) {
    int* ctr = a.counters + rb;
    const int old = atomicAdd(ctr, 1);
    hd.last = (old == units - 1);
    if (hd.last) *ctr = 0;
  }
  __syncthreads();
  if (!hd.last) return;
  __threadfence();
  for (int i = threadIdx.x; i < a.T * g.R; i += g.threads) {
    const int t = i / g.R, n = row0 + (i - t * g.R);
    float acc = 0.f;
    for (int j = 0; j < a.k; j++) {
      const int f = t * a.k + j;
      acc = fmaf(a.rec->w[f], __ldcg(a.y + (size_t)a.rec->pos[f] * a.H + n), acc);
    }
    for (int s = 0; s < a.n_shared; s++) acc += __ldcg(a.y + (size_t)(a.T * a.k + s * a.T + t) * a.H + n);
    __nv_bfloat16 b = __float2bfloat16_rn(acc);
    a.out[(size_t)t * a.H + n] = *reinterpret_cast<uint16_t*>(&b);
  }
}

// ---------------------------------------------------------------------------
// routing kernel: CTA l routes layer l and stores its record
// ---------------------------------------------------------------------------
template <int PER>
__global__ void __launch_bounds__(kThreads) k_route(RouteArgs a) {
  __shared__ Route r;
  const int l = blockIdx.x;
  route_in_cta<PER>(a.logits + (size_t)l * a.T * a.E, a.T, a.E, a.k, a.renorm, r, a.status);
  const int4* src = reinterpret_cast<const int4*>(&r);
  int4* dst = reinterpret_cast<int4*>(a.rec + l);
  for (int i = threadIdx.x; i < (int)(sizeof(Route) / 16); i += kThreads) dst[i] = src[i];
  if (l == a.n_layers - 1 && a.ids_out) {
    for (int f = threadIdx.x; f < a.T * a.k; f += kThreads) {
      a.ids_out[f] = r.ids[f];
      a.w_out[f] = r.w[f];
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t decode_smem_bytes(int K, int rows, int nmat) { return make_geo(K, rows, nmat).total; }

static cudaError_t launch_one(void (*kern)(DecodeArgs), const DecodeArgs& a, const Geo& g, int grid, bool pdl,
                              cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g.total);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute at[1];
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(g.threads);
  cfg.gridDim = dim3(grid);
  cfg.dynamicSmemBytes = g.total;
  cfg.stream = s;
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
  void (*k)(RouteArgs);
  if (a.E <= 32) k = k_route<1>;
  else if (a.E <= 64) k = k_route<2>;
  else if (a.E <= 128) k = k_route<4>;
  else if (a.E <= 256) k = k_route<8>;
  else if (a.E <= 512) k = k_route<16>;
  else k = k_route<32>;
  k<<<a.n_layers, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dec_gate_up(const DecodeArgs& a, bool pdl, cudaStream_t s) {
  const Geo g = make_geo(a.H, a.I, 2);
  return launch_one(k_dec_gate_up, a, g, (a.max_units + a.n_shared) * (a.I / g.R), pdl, s);
}

cudaError_t launch_dec_down(const DecodeArgs& a, bool pdl, cudaStream_t s) {
  const Geo g = make_geo(a.I, a.H, 1);
  return launch_one(k_dec_down, a, g, (a.max_units + a.n_shared) * (a.H / g.R), pdl, s);
}

}  // namespace ft

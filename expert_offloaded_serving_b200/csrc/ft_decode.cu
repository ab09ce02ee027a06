// Decode path for small batches (T <= 16).
//
//   k_route         one CTA per layer: softmax top-k of the T tokens and the
//                   permutation of their (token, rank) pairs by expert, stored
//                   as a compact routing record (distinct experts = units).
//   k_dec_gate_up   CTA = (unit, block of R rows of Wg and Wu) over the full K,
//                   staged in shared memory by 16-byte cp.async copies; the
//                   GEMV tile below computes both matrices' rows and SwiGLU
//                   gives fp32 h.
//   k_dec_down      CTA = (unit, block of R rows of Wd) over K = I; launched as a
//                   programmatic dependent of gate/up, so its tile streams in
//                   while gate/up runs; after griddepcontrol.wait it reads h and
//                   writes y.  The last CTA to finish a row block (an atomic
//                   counter per block) sums w[t][j] * y over j ascending plus
//                   the shared expert and rounds once to bf16.
//   k_dec_stack     persistent and cooperative: one launch runs a stack of
//                   layers; each CTA takes the gate/up and the down tiles with
//                   its index modulo the grid, layer after layer; layers hand
//                   over through bounded counters in global memory instead of
//                   kernel boundaries; same arithmetic as the two kernels above.
//                   (One or two tokens go to the dataflow kernel of
//                   ft_decode_flow.cu unless FT_STACK_COUNTERS asks for this one.)
//
// All three share the GEMV tile: lanes own 32-code chunks of K and hold their
// chunk's activations (re-encoded per 32-element block as f16) in registers,
// dots by fma.rn.f32.f16 on exact products, four rows per lane group reduced by
// a transposing shuffle tree.
//
// Pages: decode fetches or reuses the selected experts and sums their partial
// results exactly (jansverre.net, "Hvorfor er båndbredden viktigere enn antall
// kjerner?"); a gate picks a few experts per token (aiforradalom.hu, "A
// Mixture-of-Experts (MoE) kihívásai és a FreeToken megoldásai").
#include <algorithm>

#include "ft_common.cuh"
#include "ft_decode.h"
#include "ft_tile.cuh"

namespace ft {
using namespace tile;
namespace {

constexpr int kThreads = 256;       // routing kernel

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }


// ---------------------------------------------------------------------------
// routing inside a CTA
// ---------------------------------------------------------------------------
// Per-CTA shared header of the GEMV kernels, then the tiles.
struct CtaHdr {
  int32_t tok[16];
  int32_t last;
  float ts[2];  // NVFP4: the matrix scales of the tile's matrices (else unused)
  int32_t pad;
};
static_assert(sizeof(CtaHdr) <= 128, "CtaHdr");

// NVFP4: the fp32 scale of matrix `mat` (0 Wg, 1 Wu, 2 Wd) of a blob.
__device__ __forceinline__ float nv_matrix_scale(const uint8_t* blob, const BlobLayout& lay, int mat) {
  return reinterpret_cast<const float*>(blob + lay.ts)[mat];
}
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

}  // namespace

// ---------------------------------------------------------------------------
// gate/up + SwiGLU: CTA = (unit, block of R rows of Wg and Wu), full K = H
// ---------------------------------------------------------------------------
template <int F>
__global__ void __launch_bounds__(kGemvThreads, 1) k_dec_gate_up(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  CtaHdr& hd = *reinterpret_cast<CtaHdr*>(smem);
  uint8_t* base = smem + kTileOff;
  const Gv g = make_gv(a.H, a.I, 2, F);
  const int nrb = a.I / g.R;
  const int rb = blockIdx.x % nrb, u = a.n_sel ? a.sel[blockIdx.x / nrb] : blockIdx.x / nrb;
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
  stage_mat(g, base, 0, blob + a.lay.wg, blob + a.lay.wg_sf, row0);
  stage_mat(g, base, 1, blob + a.lay.wu, blob + a.lay.wu_sf, row0);
  cp_async_commit();
  if (F == kFmtNv && threadIdx.x < 2) hd.ts[threadIdx.x] = nv_matrix_scale(blob, a.lay, threadIdx.x);
  pdl_trigger();
  pdl_wait();  // x is the previous kernel's output when launched as a dependent
  const LaneMap m = lane_map(g);
  for (int t0 = 0; t0 < ui.m; t0 += kMT) {
    const int n = min(kMT, ui.m - t0);
    __syncthreads();
    stage_x<true>(g, base, a.x, hd.tok + t0, n);
    cp_async_wait_all();
    __syncthreads();
    tile_dots<F>(g, m, base, n);
    __syncthreads();
    if (threadIdx.x < g.R * n) {
      const int t = threadIdx.x >> g.rlog, r = threadIdx.x & (g.R - 1);
      float gv = row_value(g, base, 0, r, t), uv = row_value(g, base, 1, r, t);
      if (F == kFmtNv) {
        gv *= hd.ts[0];
        uv *= hd.ts[1];
      }
      a.h[(size_t)(ui.hbase + t0 + t) * a.I + row0 + r] = silu(gv) * uv;
    }
  }
}

// ---------------------------------------------------------------------------
// down + combine: CTA = (unit, block of R rows of Wd), full K = I.  The last
// CTA to finish a row block (one counter per block) does the weighted combine.
// ---------------------------------------------------------------------------
template <int F>
__global__ void __launch_bounds__(kGemvThreads, 1) k_dec_down(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  CtaHdr& hd = *reinterpret_cast<CtaHdr*>(smem);
  uint8_t* base = smem + kTileOff;
  const Gv g = make_gv(a.I, a.H, 1, F);
  const int nrb = a.H / g.R;
  const int rb = blockIdx.x % nrb, u = a.n_sel ? a.sel[blockIdx.x / nrb] : blockIdx.x / nrb;
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
  stage_mat(g, base, 0, blob + a.lay.wd, blob + a.lay.wd_sf, row0);
  cp_async_commit();
  if (F == kFmtNv && threadIdx.x == 0) hd.ts[0] = nv_matrix_scale(blob, a.lay, 2);
  pdl_trigger();
  pdl_wait();  // h is written by the gate/up kernel
  if (threadIdx.x < 16) hd.tok[threadIdx.x] = ui.hbase + threadIdx.x;  // h rows of the unit's tokens
  const LaneMap m = lane_map(g);
  for (int t0 = 0; t0 < ui.m; t0 += kMT) {
    const int n = min(kMT, ui.m - t0);
    __syncthreads();
    stage_x<false>(g, base, a.h, hd.tok + t0, n);
    cp_async_wait_all();
    __syncthreads();
    tile_dots<F>(g, m, base, n);
    __syncthreads();
    if (threadIdx.x < g.R * n) {
      const int t = threadIdx.x >> g.rlog, r = threadIdx.x & (g.R - 1);
      float yv = row_value(g, base, 0, r, t);
      if (F == kFmtNv) yv *= hd.ts[0];
      a.y[(size_t)(ui.hbase + t0 + t) * a.H + row0 + r] = yv;
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
  for (int i = threadIdx.x; i < a.T * g.R; i += kGemvThreads) {
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
// parity export: matrix `mat` of a blob dequantised through the GEMV tile.
// CTA = R rows staged exactly as the GEMV kernels stage them (stage_mat),
// then each (row, chunk) is read back with tile_chunk and its codes decoded by
// e2m1x8_to_f16x8, the conversion the dot products use; out = f16 value x
// UE8M0 scale (exact in fp32 unless it overflows).
// ---------------------------------------------------------------------------
template <int F>
__global__ void __launch_bounds__(kGemvThreads, 1) k_dec_dequant(const uint8_t* blob, BlobLayout lay, int mat, int H,
                                                                 int I, float* out) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* base = smem + kTileOff;
  const int K = mat < 2 ? H : I, rows = mat < 2 ? I : H;
  const Gv g = make_gv(K, rows, 1, F);
  const int row0 = blockIdx.x * g.R;
  const int64_t co = mat == 0 ? lay.wg : mat == 1 ? lay.wu : lay.wd;
  const int64_t so = mat == 0 ? lay.wg_sf : mat == 1 ? lay.wu_sf : lay.wd_sf;
  stage_mat(g, base, 0, blob + co, blob + so, row0);
  cp_async_commit();
  cp_async_wait_all();
  __syncthreads();
  const uint8_t* codes = base + g.codes;
  const uint32_t* sc = reinterpret_cast<const uint32_t*>(base + g.scales);
  const float ts = F == kFmtNv ? nv_matrix_scale(blob, lay, mat) : 1.f;
  for (int i = threadIdx.x; i < g.R * g.chunks; i += kGemvThreads) {
    const int r = i / g.chunks, c = i - r * g.chunks;
    float* o = out + (size_t)(row0 + r) * K + c * 32;
    if constexpr (F == kFmtBf16) {
      uint4 q[4];
      tile_chunk_bf16(g, codes, r, c, q);
#pragma unroll
      for (int i4 = 0; i4 < 4; i4++) {
        const uint32_t ws[4] = {q[i4].x, q[i4].y, q[i4].z, q[i4].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
          o[8 * i4 + 2 * j] = __uint_as_float(ws[j] << 16);
          o[8 * i4 + 2 * j + 1] = __uint_as_float(ws[j] & 0xffff0000u);
        }
      }
    } else {
      uint4 q;
      float s0, s1;
      if constexpr (F == kFmtNv) {
        tile_chunk_nv(g, codes, sc, r, c, q, s0, s1);
      } else {
        tile_chunk(g, codes, sc, r, c, q, s0);
        s1 = s0;
      }
      const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int wv = 0; wv < 4; wv++) {
        uint32_t hv[4];
        e2m1x8_to_f16x8(qs[wv], hv);
        const float s = wv < 2 ? s0 : s1;
#pragma unroll
        for (int j = 0; j < 4; j++) {
          const float2 f = f16x2_to_f32x2(hv[j]);
          // NVFP4: (code x block scale) is exact; the matrix scale rounds once
          o[8 * wv + 2 * j] = F == kFmtNv ? (f.x * s) * ts : f.x * s;
          o[8 * wv + 2 * j + 1] = F == kFmtNv ? (f.y * s) * ts : f.y * s;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// persistent stacked decode: one cooperative launch for n_layers layers
// ---------------------------------------------------------------------------
namespace {


// One tile of a layer as resolved from the routing record: resolving takes a
// chain of dependent global loads (record -> unit -> pointer table ->
// permutation), so it is done when the tile's weights are issued, ahead of
// the wait that precedes its compute.
struct TileMeta {
  const uint8_t* blob;  // NULL: the expert is missing
  int32_t m;            // tokens of the unit
  int32_t hbase;        // first h / y row of the unit
  int32_t row0;         // first weight row of the tile
  int32_t pad;
  int32_t tok[16];      // gate/up: token ids; down: h rows
};

// Shared header of the persistent kernel, followed in shared memory by
// TileMeta first[n_layers][2] (this CTA's first gate/up and first down tile
// of every layer, resolved before the first layer) and int32 units[n_layers].
struct StackHdr {
  uint64_t bar[2];      // completion of the bulk weight copies into buffers A and B
  TileMeta mx;          // a later tile of the current phase
  int32_t last;
  int32_t abort;
  int32_t pad[2];
  float cw[kMaxPairs];  // combine weights of the layer, pair order
  int32_t cpos[kMaxPairs];  // y row of each pair
};

__host__ __device__ inline size_t stack_hdr_bytes(int n_layers) {
  return sizeof(StackHdr) + (size_t)n_layers * (2 * sizeof(TileMeta) + sizeof(int32_t));
}

// Lane 0 of the last warp publishes arrivals, so that thread 0, which polls,
// goes on to its next wait without waiting for the fence.
constexpr int kArriver = kGemvThreads - 32;
// Lane 0 of warp 1 issues the bulk weight copies.
constexpr int kIssuer = 32;

// The CTA's global writes so far, then one arrival at *p (after the barrier,
// a fence by the arriving thread is cumulative over the CTA's writes).  The
// arriver's warp issues nothing more until the fence is done, so that the
// fence does not also wait for the warp's next loads; the other warps go on.
__device__ __forceinline__ void cta_arrive(int* p) {
  __syncthreads();
  if ((threadIdx.x >> 5) == (kArriver >> 5)) {
    if (threadIdx.x == kArriver) {
      fence_acq_rel();
      red_add(p, 1);
    }
    __syncwarp();
  }
}

// One warp resolves tile i of a phase (nrb row blocks of R rows per unit) of
// layer `rec` into m; the caller synchronises before the CTA reads it.
__device__ __forceinline__ void resolve_tile(const StackArgs& a, const Route* rec, const uint8_t* const* eptr, int i,
                                             int nrb, int R, bool gate_up, TileMeta& m) {
  const int u = i / nrb, n_act = rec->n_active;
  int e, cnt, hbase;
  bool shared;
  if (u < n_act) {
    e = rec->unit_e[u];
    cnt = rec->unit_m[u];
    hbase = rec->unit_p0[u];
    shared = false;
  } else {
    e = a.E + (u - n_act);
    cnt = a.T;
    hbase = a.T * a.k + (u - n_act) * a.T;
    shared = true;
  }
  const int t = threadIdx.x & 31;
  if (t < cnt) m.tok[t] = !gate_up ? hbase + t : shared ? t : rec->perm[hbase + t] / a.k;
  if (t == 0) {
    const uint8_t* blob = eptr[e];
    m.blob = blob;
    m.m = cnt;
    m.hbase = hbase;
    m.row0 = (i % nrb) * R;
    if (!blob) set_status(a.status, kStMissing);
  }
}

}  // namespace

// Each CTA walks, layer after layer, its gate/up tiles (unit x R rows of Wg and
// Wu) and then its down tiles (unit x R rows of Wd); tile i of a phase goes to
// CTA i mod gridDim.  Dependencies between CTAs go through counters in global
// memory.  Per layer: [0] gate/up tiles done (down waits for all of them);
// [1] row blocks combined; [2 + rb] down tiles done in row block rb.  The
// last down tile of a row block combines that block into the layer output
// and the next layer waits for every row block.  A CTA streams its next
// tiles' weights during a compute phase: the layer's first down tile during
// gate/up, the next layer's first gate/up tile during down.  Activations
// written by other CTAs are read from L2 only.
// HS, IS: hidden and intermediate size fixed at compile time (the tile
// geometry then folds to constants), or 0, 0 for any supported shape.
template <int HS, int IS>
__global__ void __launch_bounds__(kGemvThreads, 1) k_dec_stack(StackArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int H = HS ? HS : a.H, I = IS ? IS : a.I;
  const Gv gA = make_gv(H, I, 2), gB = make_gv(I, H, 1);
  uint8_t* baseA = smem;
  uint8_t* baseB = smem + gA.total;
  StackHdr& hd = *reinterpret_cast<StackHdr*>(smem + gA.total + gB.total);
  TileMeta* first = reinterpret_cast<TileMeta*>(&hd + 1);
  int32_t* units_of = reinterpret_cast<int32_t*>(first + 2 * a.n_layers);
  const LaneMap lmA = lane_map(gA), lmB = lane_map(gB);
  const int G = gridDim.x, b = blockIdx.x;
  const int nrbA = I / gA.R, nrbB = H / gB.R;

  // A tile's codes (R contiguous rows per matrix) arrive by bulk copies that
  // one thread issues and that complete on the buffer's mbarrier; its scale
  // words by 4-byte cp.async from every thread (one commit group per tile).
  uint32_t phase[2] = {0u, 0u};     // parity of each buffer's next phase
  bool pending[2] = {false, false};  // a tile issued into the buffer and not waited for
  auto issue_codes = [&](int buf, const Gv& g, uint8_t* base, const uint8_t* m0, const uint8_t* m1, int row0) {
    if (threadIdx.x == kIssuer) {
      const uint32_t bytes = (uint32_t)g.R * (uint32_t)(g.K / 2);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_expect_tx(&hd.bar[buf], m0 ? bytes * (m1 ? 2u : 1u) : 0u);
      if (m0) bulk_g2s(base + g.codes, m0 + (size_t)row0 * (g.K / 2), bytes, &hd.bar[buf]);
      if (m0 && m1) bulk_g2s(base + g.codes + bytes, m1 + (size_t)row0 * (g.K / 2), bytes, &hd.bar[buf]);
    }
    pending[buf] = true;
  };
  auto issue_A = [&](const TileMeta& m) {
    issue_codes(0, gA, baseA, m.blob ? m.blob + a.lay.wg : nullptr, m.blob ? m.blob + a.lay.wu : nullptr, m.row0);
    if (m.blob) {
      stage_scales(gA, baseA, 0, m.blob + a.lay.wg_sf, m.row0);
      stage_scales(gA, baseA, 1, m.blob + a.lay.wu_sf, m.row0);
    }
    cp_async_commit();
  };
  auto issue_B = [&](const TileMeta& m) {
    issue_codes(1, gB, baseB, m.blob ? m.blob + a.lay.wd : nullptr, nullptr, m.row0);
    if (m.blob) stage_scales(gB, baseB, 0, m.blob + a.lay.wd_sf, m.row0);
    cp_async_commit();
  };
  // every thread waits for buffer buf's codes; a timeout marks the CTA aborted
  auto wait_codes = [&](int buf) {
    if (!mbar_wait(&hd.bar[buf], phase[buf], a.status)) hd.abort = 1;
    phase[buf] ^= 1u;
    pending[buf] = false;
  };
  // before an early return: let the copies in flight land (bounded)
  auto drain = [&]() {
    for (int buf = 0; buf < 2; buf++)
      if (pending[buf]) mbar_wait(&hd.bar[buf], phase[buf], a.status);
    cp_async_wait_all();
  };
  auto load_combine = [&](const Route* rec) {  // combine weights and y rows of a layer
    for (int f = threadIdx.x; f < a.T * a.k; f += kGemvThreads) {
      hd.cw[f] = rec->w[f];
      hd.cpos[f] = rec->pos[f];
    }
  };

  // Before the first layer, warp w resolves layers w, w + 16, ...: their
  // units and this CTA's first tile of each phase.  Every routing record is
  // complete before the launch.
  if (threadIdx.x == 0) {
    hd.abort = 0;
    mbar_init(&hd.bar[0]);
    mbar_init(&hd.bar[1]);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int l = threadIdx.x >> 5; l < a.n_layers; l += kWarps) {
    const Route* rec = a.rec + l;
    const uint8_t* const* eptr = a.eptr + (size_t)l * a.n_blobs;
    const int un = rec->n_active + a.n_shared;
    if ((threadIdx.x & 31) == 0) units_of[l] = un;
    if (b < un * nrbA) resolve_tile(a, rec, eptr, b, nrbA, gA.R, true, first[2 * l]);
    if (b < un * nrbB) resolve_tile(a, rec, eptr, b, nrbB, gB.R, false, first[2 * l + 1]);
  }
  __syncthreads();
  int units = units_of[0];
  bool preB = b < units * nrbB;
  if (b < units * nrbA) issue_A(first[0]);
  if (preB) issue_B(first[1]);

  // Prefetch order: a layer's first down tile is issued once its gate/up
  // activations are staged, the next layer's first gate/up tile once the down
  // activations are staged, so each streams in during a compute phase, behind
  // the staging loads, and no arrival's fence runs while weight copies of
  // this CTA are in flight.
  bool issuedB = preB;  // layer 0's down tile went out at the start
  for (int l = 0; l < a.n_layers; l++) {
    const Route* rec = a.rec + l;
    const uint8_t* const* eptr = a.eptr + (size_t)l * a.n_blobs;
    const int tilesA = units * nrbA, tilesB = units * nrbB;
    const bool haveA = b < tilesA, haveB = b < tilesB;
    const uint16_t* xin = l == 0 ? a.x0 : a.xbuf[(l - 1) & 1];
    uint16_t* xout = l == a.n_layers - 1 ? a.out : a.xbuf[l & 1];
    int* sy = a.sync + (size_t)l * a.sync_stride;
    const int units_n = l + 1 < a.n_layers ? units_of[l + 1] : 0;
    const bool nextA = b < units_n * nrbA;
    // the combine weights of this layer's row-block combines
    if (haveB) load_combine(rec);
    if (haveB && !haveA && !issuedB) {
      issue_B(first[2 * l + 1]);
      issuedB = true;
    }
    // ---------------- gate/up + SwiGLU ----------------
    for (int i = b; i < tilesA; i += G) {
      if (i == b) {
        // the first tile was issued ahead: wait for the previous layer
        if (l > 0) {
          const int* prev = a.sync + (size_t)(l - 1) * a.sync_stride + 1;
          if (!cta_wait_geq(prev, nrbB, hd.abort, a.status)) {
            drain();
            return;
          }
        }
      } else {
        if (threadIdx.x < 32) resolve_tile(a, rec, eptr, i, nrbA, gA.R, true, hd.mx);
        __syncthreads();
        issue_A(hd.mx);
      }
      const TileMeta& m = i == b ? first[2 * l] : hd.mx;
      for (int t0 = 0; t0 < m.m; t0 += kMT) {
        const int n = min(kMT, m.m - t0);
        if (t0 > 0) __syncthreads();
        stage_x<true>(gA, baseA, xin, m.tok + t0, n);
        // the layer's first down tile streams in during the gate/up compute;
        // issued after the staging loads so as not to queue ahead of them
        if (i == b && t0 == 0 && haveB && !issuedB) {
          issue_B(first[2 * l + 1]);
          issuedB = true;
        }
        // the first tile's down weights were issued after it: leave them in flight
        if (i == b && haveB) cp_async_wait_1(); else cp_async_wait_all();
        if (t0 == 0) wait_codes(0);
        __syncthreads();
        if (hd.abort) {
          drain();
          return;
        }
        tile_dots<kFmtMx>(gA, lmA, baseA, n);
        __syncthreads();
        if (threadIdx.x < gA.R * n) {
          const int t = threadIdx.x >> gA.rlog, r = threadIdx.x & (gA.R - 1);
          const size_t at = (size_t)(m.hbase + t0 + t) * I + m.row0 + r;
          if (m.blob) a.h[at] = silu(row_value(gA, baseA, 0, r, t)) * row_value(gA, baseA, 1, r, t);
        }
      }
      cta_arrive(&sy[0]);
    }
    // without a down phase, the next layer's first gate/up tile goes out now
    if (!haveB && nextA) {
      __syncthreads();
      issue_A(first[2 * (l + 1)]);
    }
    // ---------------- down (+ row-block combine) ----------------
    if (haveB) {
      // every gate/up tile of this layer is done
      if (!cta_wait_geq(&sy[0], tilesA, hd.abort, a.status)) {
        drain();
        return;
      }
      for (int i = b; i < tilesB; i += G) {
        if (i != b) {
          __syncthreads();
          if (threadIdx.x < 32) resolve_tile(a, rec, eptr, i, nrbB, gB.R, false, hd.mx);
          __syncthreads();
          issue_B(hd.mx);
        }
        const TileMeta& mb = i == b ? first[2 * l + 1] : hd.mx;
        const int rb = i % nrbB;
        for (int t0 = 0; t0 < mb.m; t0 += kMT) {
          const int n = min(kMT, mb.m - t0);
          if (t0 > 0) __syncthreads();
          stage_x<false>(gB, baseB, a.h, mb.tok + t0, n);
          // buffer A is free since the gate/up phase: the next layer's first
          // gate/up tile streams in during the down compute
          if (i == b && t0 == 0 && nextA) issue_A(first[2 * (l + 1)]);
          // the next layer's gate/up weights were issued after this tile's
          if (i == b && nextA) cp_async_wait_1(); else cp_async_wait_all();
          if (t0 == 0) wait_codes(1);
          __syncthreads();
          if (hd.abort) {
            drain();
            return;
          }
          tile_dots<kFmtMx>(gB, lmB, baseB, n);
          __syncthreads();
          if (threadIdx.x < gB.R * n) {
            const int t = threadIdx.x >> gB.rlog, r = threadIdx.x & (gB.R - 1);
            a.y[(size_t)(mb.hbase + t0 + t) * H + mb.row0 + r] = mb.blob ? row_value(gB, baseB, 0, r, t) : 0.f;
          }
        }
        __syncthreads();
        if (threadIdx.x == kArriver) {
          fence_acq_rel();
          const int old = atom_add(&sy[2 + rb], 1);
          hd.last = old == units - 1;
          if (hd.last) fence_acq_rel();  // acquire the other tiles' y of this row block
        }
        __syncthreads();
        if (hd.last) {
          const int row0 = mb.row0;
          for (int q = threadIdx.x; q < a.T * gB.R; q += kGemvThreads) {
            const int t = q / gB.R, nn = row0 + (q - t * gB.R);
            float acc = 0.f;
            for (int j = 0; j < a.k; j++) {
              const int f = t * a.k + j;
              acc = fmaf(hd.cw[f], __ldcg(a.y + (size_t)hd.cpos[f] * H + nn), acc);
            }
            for (int s2 = 0; s2 < a.n_shared; s2++)
              acc += __ldcg(a.y + (size_t)(a.T * a.k + s2 * a.T + t) * H + nn);
            __nv_bfloat16 bb = __float2bfloat16_rn(acc);
            xout[(size_t)t * H + nn] = *reinterpret_cast<uint16_t*>(&bb);
          }
          cta_arrive(&sy[1]);
        }
      }
    }
    issuedB = false;
    units = units_n;
  }
  cp_async_wait_all();
}

// ---------------------------------------------------------------------------
// failure injection: the persistent kernel's bounded wait on a flag nothing sets
// ---------------------------------------------------------------------------
__global__ void k_debug_wait(const int* flag, int* status, uint64_t limit_ns) {
  __shared__ int abort;
  if (threadIdx.x == 0) abort = 0;
  __syncthreads();
  cta_wait_geq(flag, 1, abort, status, limit_ns);
}

// ---------------------------------------------------------------------------
// routing kernel: CTA l routes layer l and stores its record
// ---------------------------------------------------------------------------
template <int PER>
__global__ void __launch_bounds__(kThreads) k_route(RouteArgs a) {
  __shared__ Route r;
  const int l = blockIdx.x;
  route_in_cta<PER>(a.logits + (size_t)l * (a.layer_stride ? a.layer_stride : (int64_t)a.T * a.E), a.T, a.E, a.k,
                    a.renorm, r, a.status);
  const int4* src = reinterpret_cast<const int4*>(&r);
  int4* dst = reinterpret_cast<int4*>(a.rec + l);
  for (int i = threadIdx.x; i < (int)(sizeof(Route) / 16); i += kThreads) dst[i] = src[i];
  if (a.sync)
    for (int i = threadIdx.x; i < a.sync_stride; i += kThreads) a.sync[(size_t)l * a.sync_stride + i] = 0;
  if (a.epoch && l == 0) {
    // tags (e << 7 | layer) never equal a zeroed word's; when they wrap (every
    // 2^25 launches) the tagged words are zeroed, so that no word left from
    // 2^25 launches ago can carry a tag of this launch
    __shared__ int wrapped;
    if (threadIdx.x == 0) {
      bool w;
      *a.epoch = next_epoch(*a.epoch, &w);
      wrapped = w;
    }
    __syncthreads();
    if (wrapped)
      for (int64_t i = threadIdx.x; i < a.tagged_words; i += kThreads) a.tagged[i] = 0ull;
  }
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
static cudaError_t launch_one(void (*kern)(DecodeArgs), const DecodeArgs& a, const Gv& g, int rows, int grid,
                              bool pdl, cudaStream_t s) {
  if (!gv_ok(g, rows)) return cudaErrorInvalidValue;
  const size_t smem = kTileOff + g.total;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute at[1];
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(kGemvThreads);
  cfg.gridDim = dim3(grid);
  cfg.dynamicSmemBytes = smem;
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
  const int F = a.lay.fmt;
  const Gv g = make_gv(a.H, a.I, 2, F);
  const int units = a.n_sel ? a.n_sel : a.max_units + a.n_shared;
  void (*kern)(DecodeArgs) =
      F == kFmtNv ? k_dec_gate_up<kFmtNv> : F == kFmtBf16 ? k_dec_gate_up<kFmtBf16> : k_dec_gate_up<kFmtMx>;
  return launch_one(kern, a, g, a.I, units * (a.I / g.R), pdl, s);
}

cudaError_t launch_dec_down(const DecodeArgs& a, bool pdl, cudaStream_t s) {
  const int F = a.lay.fmt;
  const Gv g = make_gv(a.I, a.H, 1, F);
  const int units = a.n_sel ? a.n_sel : a.max_units + a.n_shared;
  void (*kern)(DecodeArgs) = F == kFmtNv ? k_dec_down<kFmtNv> : F == kFmtBf16 ? k_dec_down<kFmtBf16> : k_dec_down<kFmtMx>;
  return launch_one(kern, a, g, a.H, units * (a.H / g.R), pdl, s);
}

cudaError_t launch_dec_dequant(const uint8_t* blob, const BlobLayout& lay, int mat, int H, int I, float* out,
                               cudaStream_t s) {
  const int K = mat < 2 ? H : I, rows = mat < 2 ? I : H;
  const Gv g = make_gv(K, rows, 1, lay.fmt);
  if (!gv_ok(g, rows)) return cudaErrorInvalidValue;
  const size_t smem = kTileOff + g.total;
  void (*kern)(const uint8_t*, BlobLayout, int, int, int, float*) =
      lay.fmt == kFmtNv ? k_dec_dequant<kFmtNv> : lay.fmt == kFmtBf16 ? k_dec_dequant<kFmtBf16> : k_dec_dequant<kFmtMx>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<rows / g.R, kGemvThreads, smem, s>>>(blob, lay, mat, H, I, out);
  return cudaGetLastError();
}

bool decode_supported(int H, int I, int fmt) {
  return gv_ok(make_gv(H, I, 2, fmt), I) && gv_ok(make_gv(I, H, 1, fmt), H);
}

void decode_geometry(int H, int I, int64_t* out) {
  const Gv gs[2] = {make_gv(H, I, 2), make_gv(I, H, 1)};
  const int rows[2] = {I, H};
  for (int p = 0; p < 2; p++) {
    const Gv& g = gs[p];
    int64_t* o = out + 10 * p;
    o[0] = g.K;
    o[1] = g.chunks;
    o[2] = g.lpr;
    o[3] = g.rpw;
    o[4] = g.parts;
    o[5] = g.rsets;
    o[6] = g.groups;
    o[7] = g.R;
    o[8] = (int64_t)(kTileOff + g.total);
    o[9] = gv_ok(g, rows[p]) ? 1 : 0;
  }
  out[20] = kGemvThreads;
  out[21] = (int64_t)kSmemLimit;
}

constexpr size_t kStackSmemMax = 227 * 1024;  // opt-in dynamic shared memory per CTA

bool stack_supported(int H, int I, int n_layers) {
  const Gv gA = make_gv(H, I, 2), gB = make_gv(I, H, 1);
  return gv_ok(gA, I) && gv_ok(gB, H) && gA.total + gB.total + stack_hdr_bytes(n_layers) <= kStackSmemMax;
}

cudaError_t launch_debug_wait(const int* flag, int* status, uint64_t limit_ns, cudaStream_t s) {
  k_debug_wait<<<1, 32, 0, s>>>(flag, status, limit_ns);
  return cudaGetLastError();
}

int stack_sync_stride(int H, int I) { return 2 + H / make_gv(I, H, 1).R; }

cudaError_t launch_dec_stack(const StackArgs& a, cudaStream_t s) {
  if (!stack_supported(a.H, a.I, a.n_layers) || a.sync_stride < stack_sync_stride(a.H, a.I))
    return cudaErrorInvalidValue;
  const Gv gA = make_gv(a.H, a.I, 2), gB = make_gv(a.I, a.H, 1);
  const size_t smem = gA.total + gB.total + stack_hdr_bytes(a.n_layers);
  // the 35B-class shape (hidden 2048, intermediate 512) has its own build
  void (*kern)(StackArgs) = (a.H == 2048 && a.I == 512) ? k_dec_stack<2048, 512> : k_dec_stack<0, 0>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0, occ = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
      (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGemvThreads, smem)) != cudaSuccess)
    return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  // no layer has more tiles than (distinct experts + shared) x row blocks
  const int units_max = std::min(a.E, a.T * a.k) + a.n_shared;
  const int tiles_max = units_max * std::max(a.I / gA.R, a.H / gB.R);
  const int grid = std::min(nsm * occ, tiles_max);
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(kGemvThreads);
  cfg.gridDim = dim3(grid);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace ft

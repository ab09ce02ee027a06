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
//                   over through bounded counters in global memory (and, for
//                   one or two tokens, h through tagged words) instead of
//                   kernel boundaries; same arithmetic as the two kernels above.
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

namespace ft {
namespace {

constexpr int kThreads = 256;       // routing kernel
constexpr int kGemvThreads = 512;   // GEMV kernels

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

// ---------------------------------------------------------------------------
// GEMV tile (host and device).  A CTA of kGemvThreads threads takes R
// consecutive weight rows of nmat matrices over the full K of one unit.  K is
// cut into chunks of 32 codes (16 bytes under one UE8M0 scale).  A lane owns
// one chunk: it holds that chunk's activations of up to kMT tokens in
// registers and takes the chunk in every row given to its lane group.  A lane
// group is lpr lanes (a power of two) on lpr consecutive chunks; rpw = 32/lpr
// groups share a warp; when K has more than 32 chunks, `parts` groups side by
// side cover it (warp w takes part w % parts).
//
// Arithmetic.  The activations of a pass are first re-encoded in shared
// memory as f16 with one power-of-two factor per 32-element block, chosen so
// that the block's largest magnitude lands in [2^14, 2^15): a bf16 x is
// re-encoded exactly (down to 2^-28 of its block's largest element), an fp32 h
// is rounded to 11 significant bits.  A weight code becomes f16 exactly
// (cvt.rn.f16x2.e2m1x2), each product w*x is exact in fp32, and the 32 terms
// of a chunk are summed by fp32 fused multiply-adds (fma.rn.f32.f16) in a fixed
// order into two accumulators; the chunk's value is that sum times (weight
// scale x inverse activation factor).  A row's value is the sum of its
// chunks' values: the lanes of a group add theirs with xor shuffles, then the
// parts are added in ascending order through shared memory.
//
// Shared memory, from the tile's base:
//   codes  [nmat][R][K/2]        as in global memory (16-byte cp.async copies)
//   scales [nmat][R][K/128]      words of four blocks' UE8M0 bytes
//   xh     [kMT][4][K/32] x 16 B  activations, f16: quad i of chunk c at [t][i][c]
//   xinv   [kMT][K/32]           inverse block factors
//   red    [parts][nmat][R][kMT] partial sums
// ---------------------------------------------------------------------------
constexpr int kMT = 2;                      // tokens per pass over the tile
constexpr int kWarps = kGemvThreads / 32;
constexpr size_t kSmemLimit = 220 * 1024;
constexpr size_t kTileBytes = 64 * 1024;    // weight codes per tile, about

struct Gv {
  int K, chunks, atoms;
  int lpr, rpw, parts, rsets, groups;
  int R, rlog, nmat;  // rows per tile, a power of two (R = 1 << rlog)
  size_t codes, scales, xh, xinv, red, total;
};

__host__ __device__ inline Gv make_gv(int K, int rows, int nmat) {
  Gv g;
  g.K = K;
  g.nmat = nmat;
  g.chunks = K / 32;
  g.atoms = K / 128;
  g.lpr = 1;
  while (g.lpr < 32 && g.lpr < g.chunks) g.lpr <<= 1;
  g.rpw = 32 / g.lpr;
  g.parts = (g.chunks + g.lpr - 1) / g.lpr;
  g.rsets = kWarps / g.parts;  // 0 for K > 16384: not supported
  g.groups = g.rsets * g.rpw;
  int R = 128;
  while (R > 8 && (size_t)R * nmat * K / 2 > kTileBytes) R >>= 1;
  if (R > rows) R = rows;
  for (;;) {
    g.codes = 0;
    g.scales = (size_t)nmat * R * K / 2;
    g.xh = g.scales + (size_t)nmat * R * g.atoms * 4;
    g.xinv = g.xh + (size_t)kMT * K * 2;
    g.red = g.xinv + (((size_t)kMT * g.chunks * 4 + 15) & ~(size_t)15);
    g.total = g.red + (size_t)g.parts * nmat * R * kMT * 4;
    if (g.total <= kSmemLimit || R <= 8) break;
    R >>= 1;
  }
  g.R = R;
  g.rlog = 0;
  while ((1 << g.rlog) < R) g.rlog++;
  return g;
}

// Shapes the decode kernels take: K and rows multiples of 128, K <= 16384.
__host__ __device__ inline bool gv_ok(const Gv& g, int rows) {
  return g.rsets > 0 && g.total <= kSmemLimit && rows % g.R == 0;
}

// This thread's place in the tile.
struct LaneMap {
  int c;      // chunk (>= chunks: the lane holds no chunk and adds zeros)
  int grp;    // lane group: rows grp, grp + groups, ...
  int part;   // K part
  bool on;    // the warp has a row set
  bool lead;  // first lane of its group
};

__device__ __forceinline__ LaneMap lane_map(const Gv& g) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  LaneMap m;
  m.part = w % g.parts;
  const int rs = w / g.parts;
  m.on = rs < g.rsets;
  m.c = m.part * g.lpr + (lane & (g.lpr - 1));
  m.grp = rs * g.rpw + lane / g.lpr;
  m.lead = (lane & (g.lpr - 1)) == 0;
  return m;
}

// Scale words of rows [row0, row0 + R) of matrix `mat` (scale region sc_g),
// one 4-byte cp.async each.
__device__ __forceinline__ void stage_scales(const Gv& g, uint8_t* base, int mat, const uint8_t* sc_g, int row0) {
  uint32_t* sd = reinterpret_cast<uint32_t*>(base + g.scales) + (size_t)mat * g.R * g.atoms;
  for (int i = threadIdx.x; i < g.R * g.atoms; i += kGemvThreads) {
    const int r = i / g.atoms, at = i - r * g.atoms;
    cp_async4(sd + i, sc_g + sf_word(row0 + r, at, g.atoms));
  }
}

// Stage rows [row0, row0 + R) of matrix `mat` (codes at codes_g, row pitch
// K/2; scale region sc_g) into the tile with cp.async.
__device__ __forceinline__ void stage_mat(const Gv& g, uint8_t* base, int mat, const uint8_t* codes_g,
                                          const uint8_t* sc_g, int row0) {
  uint8_t* dst = base + g.codes + (size_t)mat * g.R * (g.K / 2);
  const uint8_t* src = codes_g + (size_t)row0 * (g.K / 2);
  const int n16 = g.R * g.chunks;
  for (int i = threadIdx.x; i < n16; i += kGemvThreads) cp_async16(dst + (size_t)i * 16, src + (size_t)i * 16);
  stage_scales(g, base, mat, sc_g, row0);
}

// Encode 4 consecutive activations v (group q of token t) into the tile's f16
// activations; the 8 lanes of a 32-element block agree on its factor by
// shuffles, so all 32 lanes of the warp must call this together.
__device__ __forceinline__ void encode4(const Gv& g, uint8_t* base, int t, int q, const float (&v)[4]) {
  uint2* xh = reinterpret_cast<uint2*>(base + g.xh);
  float* xinv = reinterpret_cast<float*>(base + g.xinv);
  uint32_t e = 0;
#pragma unroll
  for (int j = 0; j < 4; j++) e = max(e, __float_as_uint(v[j]) & 0x7f800000u);
  e = max(e, __shfl_xor_sync(0xffffffffu, e, 1));
  e = max(e, __shfl_xor_sync(0xffffffffu, e, 2));
  e = max(e, __shfl_xor_sync(0xffffffffu, e, 4));
  // largest biased exponent of the block, at least 15 so that both factors
  // are normal floats: 2^(141-eb) maps the block's maximum into [2^14, 2^15)
  const int eb = max((int)(e >> 23), 15);
  const float f = __uint_as_float((uint32_t)(268 - eb) << 23);
  __half2 h0 = __float22half2_rn(make_float2(v[0] * f, v[1] * f));
  __half2 h1 = __float22half2_rn(make_float2(v[2] * f, v[3] * f));
  // quad i (16 bytes) of chunk c sits at [t][i][c], so that the lanes of a
  // warp, one chunk each, read consecutive 16-byte words
  const int c = q >> 3, i = (q & 7) >> 1;
  xh[(size_t)t * (g.K / 4) + 2 * ((size_t)i * g.chunks + c) + (q & 1)] =
      make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
  if ((q & 7) == 0) xinv[t * g.chunks + c] = __uint_as_float((uint32_t)(eb - 14) << 23);
}

// Re-encode tokens rows[0 .. n) of a bf16 (x) or fp32 (h) matrix with row
// length K into the tile's f16 activations (read from L2).  Thread i takes 4
// consecutive elements.  With n > 1, tokens n .. kMT-1 are zero.
template <bool BF16>
__device__ __forceinline__ void stage_x(const Gv& g, uint8_t* base, const void* src, const int* rows, int n) {
  const int per = g.K / 4;
  // tokens n .. kMT-1 are staged only when a pass reads them (n > 1); the
  // bound is a multiple of 32, so a warp is wholly inside or outside
  const int items = (n > 1 ? kMT : 1) * per;
  for (int i = threadIdx.x; i < items; i += kGemvThreads) {
    const int t = i / per, q = i - t * per;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (t < n) {
      if (BF16) {
        const uint2 w = __ldcg(reinterpret_cast<const uint2*>((const uint16_t*)src + (size_t)rows[t] * g.K) + q);
        v[0] = __uint_as_float(w.x << 16);
        v[1] = __uint_as_float(w.x & 0xffff0000u);
        v[2] = __uint_as_float(w.y << 16);
        v[3] = __uint_as_float(w.y & 0xffff0000u);
      } else {
        const float4 u = __ldcg(reinterpret_cast<const float4*>((const float*)src + (size_t)rows[t] * g.K) + q);
        v[0] = u.x;
        v[1] = u.y;
        v[2] = u.z;
        v[3] = u.w;
      }
    }
    encode4(g, base, t, q, v);
  }
}

// Two e2m1 codes per byte of w -> four f16 pairs (byte b: elements 2b, 2b+1).
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t (&h)[4]) {
  asm("{ .reg .b8 b0, b1, b2, b3; mov.b32 {b0, b1, b2, b3}, %4;"
      " cvt.rn.f16x2.e2m1x2 %0, b0; cvt.rn.f16x2.e2m1x2 %1, b1;"
      " cvt.rn.f16x2.e2m1x2 %2, b2; cvt.rn.f16x2.e2m1x2 %3, b3; }"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(w));
}

// acc += w.lo * x.lo, then acc += w.hi * x.hi (f16 operands, fp32 fused).
__device__ __forceinline__ float fma_f16x2(uint32_t w, uint32_t x, float acc) {
  asm("{ .reg .f16 wl, wh, xl, xh; mov.b32 {wl, wh}, %1; mov.b32 {xl, xh}, %2;"
      " fma.rn.f32.f16 %0, wl, xl, %0; fma.rn.f32.f16 %0, wh, xh, %0; }"
      : "+f"(acc) : "r"(w), "r"(x));
  return acc;
}

// Codes (16 bytes, 32 e2m1 values) and decoded UE8M0 scale of chunk c of
// staged row `row` (rows of all matrices of the tile counted in order).
__device__ __forceinline__ void tile_chunk(const Gv& g, const uint8_t* codes, const uint32_t* sc, int row, int c,
                                           uint4& q, float& s) {
  q = *reinterpret_cast<const uint4*>(codes + (size_t)row * (g.K / 2) + c * 16);
  const uint32_t sw = sc[(size_t)row * g.atoms + (c >> 2)];
  s = ue8m0_to_f32((sw >> (8 * (c & 3))) & 0xffu);
}

// Dot of one chunk of 32 e2m1 codes with NT tokens' f16 activations x[t][i]
// (elements 2i, 2i+1); even code bytes feed one accumulator, odd ones the
// other.
template <int NT>
__device__ __forceinline__ void chunk_dot(uint4 q, const uint32_t (&x)[kMT][16], float* d) {
  float acc[NT][2];
#pragma unroll
  for (int t = 0; t < NT; t++) acc[t][0] = acc[t][1] = 0.f;
  const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int wv = 0; wv < 4; wv++) {
    uint32_t h[4];
    e2m1x8_to_f16x8(qs[wv], h);
#pragma unroll
    for (int j = 0; j < 4; j++)
#pragma unroll
      for (int t = 0; t < NT; t++) acc[t][j & 1] = fma_f16x2(h[j], x[t][4 * wv + j], acc[t][j & 1]);
  }
#pragma unroll
  for (int t = 0; t < NT; t++) d[t] = acc[t][0] + acc[t][1];
}

// Sum over the lpr lanes of a group of RU rows' partial sums v[u][t] (RU = 1,
// 2 or 4, RU <= lpr).  The first one or two xor steps exchange halves of the
// rows (each lane keeps the half its lane bit selects) and the remaining
// steps add; afterwards row u's sum is on the lanes whose two group-lane bits
// (lpr/2, lpr/4) spell u and whose lower bits are zero.  Returns that row.
template <int RU, int NT>
__device__ __forceinline__ int group_reduce(float (&v)[4][kMT], int lpr) {
  const int lane = threadIdx.x & 31;
  int row = 0, d = lpr >> 1;
  if (RU == 4) {
    const bool hi = lane & d;
#pragma unroll
    for (int t = 0; t < NT; t++) {
      const float s0 = hi ? v[0][t] : v[2][t], s1 = hi ? v[1][t] : v[3][t];
      const float k0 = hi ? v[2][t] : v[0][t], k1 = hi ? v[3][t] : v[1][t];
      v[0][t] = k0 + __shfl_xor_sync(0xffffffffu, s0, d);
      v[1][t] = k1 + __shfl_xor_sync(0xffffffffu, s1, d);
    }
    row = hi ? 2 : 0;
    d >>= 1;
  }
  if (RU >= 2) {
    const bool hi = lane & d;
#pragma unroll
    for (int t = 0; t < NT; t++) {
      const float sd = hi ? v[0][t] : v[1][t], kp = hi ? v[1][t] : v[0][t];
      v[0][t] = kp + __shfl_xor_sync(0xffffffffu, sd, d);
    }
    row += hi ? 1 : 0;
    d >>= 1;
  }
  for (; d >= 1; d >>= 1)
#pragma unroll
    for (int t = 0; t < NT; t++) v[0][t] += __shfl_xor_sync(0xffffffffu, v[0][t], d);
  return row;
}

// Partial sums of the staged tile's rows for NT tokens into red.  Lane group
// grp takes rows grp + j*groups, RU of them at a time.
template <int RU, int NT>
__device__ __forceinline__ void tile_dots_t(const Gv& g, const LaneMap& m, uint8_t* base,
                                            const uint32_t (&x)[kMT][16], const float (&xi)[kMT]) {
  const uint8_t* codes = base + g.codes;
  const uint32_t* sc = reinterpret_cast<const uint32_t*>(base + g.scales);
  float* red = reinterpret_cast<float*>(base + g.red);
  const bool cv = m.c < g.chunks;
  const int lmask = RU == 4 ? (g.lpr >> 2) - 1 : RU == 2 ? (g.lpr >> 1) - 1 : g.lpr - 1;
  for (int mat = 0; mat < g.nmat; mat++) {
    // the trip count is the same for every lane of a warp, so the shuffles
    // see the whole warp
    for (int j0 = 0; m.grp + j0 * g.groups < g.R; j0 += RU) {
      float v[4][kMT];
#pragma unroll
      for (int u = 0; u < RU; u++) {
        v[u][0] = v[u][1] = 0.f;
        if (cv) {
          const int row = mat * g.R + m.grp + (j0 + u) * g.groups;
          uint4 q;
          float s;
          tile_chunk(g, codes, sc, row, m.c, q, s);
          float d[NT];
          chunk_dot<NT>(q, x, d);
#pragma unroll
          for (int t = 0; t < NT; t++) v[u][t] = d[t] * (s * xi[t]);
        }
      }
      const int u = group_reduce<RU, NT>(v, g.lpr);
      if (((threadIdx.x & 31) & lmask) == 0) {
        const int r = m.grp + (j0 + u) * g.groups;
        float* o = red + ((size_t)(m.part * g.nmat + mat) * g.R + r) * kMT;
#pragma unroll
        for (int t = 0; t < NT; t++) o[t] = v[0][t];
      }
    }
  }
}

// Partial sums of every row of the staged tile for n (<= kMT) tokens into red.
__device__ __forceinline__ void tile_dots(const Gv& g, const LaneMap& m, uint8_t* base, int n) {
  if (!m.on) return;
  uint32_t x[kMT][16];
  float xi[kMT] = {0.f, 0.f};
  if (m.c < g.chunks) {
    const uint4* xh = reinterpret_cast<const uint4*>(base + g.xh);
    const float* xinv = reinterpret_cast<const float*>(base + g.xinv);
#pragma unroll
    for (int t = 0; t < kMT; t++) {
      if (t < n) {
#pragma unroll
        for (int i = 0; i < 4; i++) {
          const uint4 u = xh[(size_t)t * (g.K / 8) + (size_t)i * g.chunks + m.c];
          x[t][4 * i] = u.x;
          x[t][4 * i + 1] = u.y;
          x[t][4 * i + 2] = u.z;
          x[t][4 * i + 3] = u.w;
        }
        xi[t] = xinv[t * g.chunks + m.c];
      } else {
#pragma unroll
        for (int i = 0; i < 16; i++) x[t][i] = 0u;
      }
    }
  } else {
#pragma unroll
    for (int t = 0; t < kMT; t++)
#pragma unroll
      for (int i = 0; i < 16; i++) x[t][i] = 0u;
  }
  // rows per lane group and matrix; groups of 4 or 2 when they divide it
  const int per = g.R % g.groups == 0 ? g.R / g.groups : 0;
  const int ru = (per % 4 == 0 && per > 0 && g.lpr >= 4) ? 4 : (per % 2 == 0 && per > 0 && g.lpr >= 2) ? 2 : 1;
  if (n > 1) {
    if (ru == 4) tile_dots_t<4, 2>(g, m, base, x, xi);
    else if (ru == 2) tile_dots_t<2, 2>(g, m, base, x, xi);
    else tile_dots_t<1, 2>(g, m, base, x, xi);
  } else {
    if (ru == 4) tile_dots_t<4, 1>(g, m, base, x, xi);
    else if (ru == 2) tile_dots_t<2, 1>(g, m, base, x, xi);
    else tile_dots_t<1, 1>(g, m, base, x, xi);
  }
}

// Row r of matrix mat for token t: the parts' partial sums in ascending order.
__device__ __forceinline__ float row_value(const Gv& g, const uint8_t* base, int mat, int r, int t) {
  const float* red = reinterpret_cast<const float*>(base + g.red);
  float s = red[((size_t)mat * g.R + r) * kMT + t];
  for (int p = 1; p < g.parts; p++) s += red[((size_t)(p * g.nmat + mat) * g.R + r) * kMT + t];
  return s;
}

}  // namespace

// ---------------------------------------------------------------------------
// gate/up + SwiGLU: CTA = (unit, block of R rows of Wg and Wu), full K = H
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kGemvThreads, 1) k_dec_gate_up(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  CtaHdr& hd = *reinterpret_cast<CtaHdr*>(smem);
  uint8_t* base = smem + kTileOff;
  const Gv g = make_gv(a.H, a.I, 2);
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
  stage_mat(g, base, 0, blob + a.lay.wg, blob + a.lay.wg_sf, row0);
  stage_mat(g, base, 1, blob + a.lay.wu, blob + a.lay.wu_sf, row0);
  cp_async_commit();
  pdl_trigger();
  pdl_wait();  // x is the previous kernel's output when launched as a dependent
  const LaneMap m = lane_map(g);
  for (int t0 = 0; t0 < ui.m; t0 += kMT) {
    const int n = min(kMT, ui.m - t0);
    __syncthreads();
    stage_x<true>(g, base, a.x, hd.tok + t0, n);
    cp_async_wait_all();
    __syncthreads();
    tile_dots(g, m, base, n);
    __syncthreads();
    if (threadIdx.x < g.R * n) {
      const int t = threadIdx.x >> g.rlog, r = threadIdx.x & (g.R - 1);
      a.h[(size_t)(ui.hbase + t0 + t) * a.I + row0 + r] =
          silu(row_value(g, base, 0, r, t)) * row_value(g, base, 1, r, t);
    }
  }
}

// ---------------------------------------------------------------------------
// down + combine: CTA = (unit, block of R rows of Wd), full K = I.  The last
// CTA to finish a row block (one counter per block) does the weighted combine.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kGemvThreads, 1) k_dec_down(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  CtaHdr& hd = *reinterpret_cast<CtaHdr*>(smem);
  uint8_t* base = smem + kTileOff;
  const Gv g = make_gv(a.I, a.H, 1);
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
  stage_mat(g, base, 0, blob + a.lay.wd, blob + a.lay.wd_sf, row0);
  cp_async_commit();
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
    tile_dots(g, m, base, n);
    __syncthreads();
    if (threadIdx.x < g.R * n) {
      const int t = threadIdx.x >> g.rlog, r = threadIdx.x & (g.R - 1);
      a.y[(size_t)(ui.hbase + t0 + t) * a.H + row0 + r] = row_value(g, base, 0, r, t);
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
__global__ void __launch_bounds__(kGemvThreads, 1) k_dec_dequant(const uint8_t* blob, BlobLayout lay, int mat, int H,
                                                                 int I, float* out) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* base = smem + kTileOff;
  const int K = mat < 2 ? H : I, rows = mat < 2 ? I : H;
  const Gv g = make_gv(K, rows, 1);
  const int row0 = blockIdx.x * g.R;
  const int64_t co = mat == 0 ? lay.wg : mat == 1 ? lay.wu : lay.wd;
  const int64_t so = mat == 0 ? lay.wg_sf : mat == 1 ? lay.wu_sf : lay.wd_sf;
  stage_mat(g, base, 0, blob + co, blob + so, row0);
  cp_async_commit();
  cp_async_wait_all();
  __syncthreads();
  const uint8_t* codes = base + g.codes;
  const uint32_t* sc = reinterpret_cast<const uint32_t*>(base + g.scales);
  for (int i = threadIdx.x; i < g.R * g.chunks; i += kGemvThreads) {
    const int r = i / g.chunks, c = i - r * g.chunks;
    uint4 q;
    float s;
    tile_chunk(g, codes, sc, r, c, q, s);
    const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
    float* o = out + (size_t)(row0 + r) * K + c * 32;
#pragma unroll
    for (int wv = 0; wv < 4; wv++) {
      uint32_t hv[4];
      e2m1x8_to_f16x8(qs[wv], hv);
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const float2 f = f16x2_to_f32x2(hv[j]);
        o[8 * wv + 2 * j] = f.x * s;
        o[8 * wv + 2 * j + 1] = f.y * s;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// persistent stacked decode: one cooperative launch for n_layers layers
// ---------------------------------------------------------------------------
namespace {

constexpr uint64_t kSpinNs = 2000ull * 1000 * 1000;  // a dependency wait gives up after 2 s

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

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t gclock() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void fence_acq_rel() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ void red_add(int* p, int v) {
  asm volatile("red.relaxed.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int atom_add(int* p, int v) {
  int old;
  asm volatile("atom.relaxed.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint64_t* bar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
               : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait for the phase with this parity; false (and the timeout status
// bit) when it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = gclock();
  while (!mbar_try(bar, parity)) {
    if (gclock() - t0 > kSpinNs) {
      set_status(status, kStTimeout);
      return false;
    }
  }
  return true;
}
// One contiguous global -> shared copy by the bulk-copy engine, completing on bar.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Thread 0 waits (acquire, bounded by limit_ns) until *p >= target, then the
// CTA synchronises; false (and the timeout status bit) when the wait gave up.
// `abort` is a shared flag, zero until a wait of this CTA gives up.
__device__ bool cta_wait_geq(const int* p, int target, int& abort, int* status, uint64_t limit_ns = kSpinNs) {
  if (threadIdx.x == 0 && ld_acquire(p) < target) {
    const uint64_t t0 = gclock();
    while (ld_acquire(p) < target) {
      if (gclock() - t0 > limit_ns) {
        set_status(status, kStTimeout);
        abort = 1;
        break;
      }
      __nanosleep(20);
    }
  }
  __syncthreads();
  return abort == 0;
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

// out[t][n] = bf16( sum_j w[t][j] * y[pos[t][j]][n]  (j ascending, fused)
//                   + sum_s y[T*k + s*T + t][n] ) for 4 consecutive n (group q)
// of row length H; the same arithmetic as the combine of the per-layer kernels.
__device__ __forceinline__ void combine4(const float* y, const float* cw, const int* cpos, int tok, int q, int H, int T,
                                         int k, int S, float (&v)[4]) {
  constexpr int kBatch = 8;  // rows in flight at once
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  // the shared expert's row is loaded with the first batch and added last
  float4 sh = make_float4(0.f, 0.f, 0.f, 0.f);
  if (S > 0) sh = __ldcg(reinterpret_cast<const float4*>(y + (size_t)(T * k + tok) * H) + q);
  for (int j0 = 0; j0 < k; j0 += kBatch) {
    float4 u[kBatch];
    float w[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; j++) {
      if (j0 + j < k) {
        const int f = tok * k + j0 + j;
        w[j] = cw[f];
        u[j] = __ldcg(reinterpret_cast<const float4*>(y + (size_t)cpos[f] * H) + q);
      }
    }
#pragma unroll
    for (int j = 0; j < kBatch; j++) {
      if (j0 + j < k) {
        acc[0] = fmaf(w[j], u[j].x, acc[0]);
        acc[1] = fmaf(w[j], u[j].y, acc[1]);
        acc[2] = fmaf(w[j], u[j].z, acc[2]);
        acc[3] = fmaf(w[j], u[j].w, acc[3]);
      }
    }
  }
  for (int s2 = 0; s2 < S; s2++) {
    const float4 u = s2 == 0 ? sh : __ldcg(reinterpret_cast<const float4*>(y + (size_t)(T * k + s2 * T + tok) * H) + q);
    acc[0] += u.x;
    acc[1] += u.y;
    acc[2] += u.z;
    acc[3] += u.w;
  }
#pragma unroll
  for (int e = 0; e < 4; e++) v[e] = __bfloat162float(__float2bfloat16_rn(acc[e]));
}

// The gate/up activations of tokens toks[0 .. n) rebuilt from the previous
// layer's y (the layer input is that layer's combined output), re-encoded like
// stage_x.
__device__ __forceinline__ void stage_comb(const Gv& g, uint8_t* base, const StackArgs& a, int H, const float* cw,
                                           const int* cpos, const int* toks, int n) {
  const int per = g.K / 4;
  const int items = (n > 1 ? kMT : 1) * per;
  for (int i = threadIdx.x; i < items; i += kGemvThreads) {
    const int t = i / per, q = i - t * per;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (t < n) combine4(a.y, cw, cpos, toks[t], q, H, a.T, a.k, a.n_shared, v);
    encode4(g, base, t, q, v);
  }
}

// h of the fused mode travels as 64-bit words (tag << 32 | fp32 bits), each
// stored and loaded whole (single-copy atomic), so a reader that sees this
// layer's tag sees the value that came with it.
__device__ __forceinline__ void st_tagged(uint64_t* p, float v, uint32_t tag) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(((uint64_t)tag << 32) | __float_as_uint(v))
               : "memory");
}
__device__ __forceinline__ void ld_tagged4(const uint64_t* p, uint64_t (&w)[4]) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(w[0]), "=l"(w[1]) : "l"(p) : "memory");
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(w[2]), "=l"(w[3]) : "l"(p + 2) : "memory");
}

// The down tile's activations from the tagged h: a word whose tag is not
// this layer's has not arrived yet and is read again, for at most 2 s (then
// the timeout bit and the CTA's abort flag are set).  Re-encoded like
// stage_x.
__device__ __forceinline__ void stage_h_tagged(const Gv& g, uint8_t* base, const uint64_t* ht, const int* rows, int n,
                                               uint32_t tag, int& abort, int* status) {
  const int per = g.K / 4;
  const int items = (n > 1 ? kMT : 1) * per;
  for (int i = threadIdx.x; i < items; i += kGemvThreads) {
    const int t = i / per, q = i - t * per;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (t < n) {
      const uint64_t* p = ht + (size_t)rows[t] * g.K + 4 * q;
      uint64_t w[4];
      ld_tagged4(p, w);
      auto ready = [&]() {
        return (uint32_t)(w[0] >> 32) == tag && (uint32_t)(w[1] >> 32) == tag && (uint32_t)(w[2] >> 32) == tag &&
               (uint32_t)(w[3] >> 32) == tag;
      };
      if (!ready()) {
        const uint64_t t0 = gclock();
        for (;;) {
          __nanosleep(20);
          ld_tagged4(p, w);
          if (ready()) break;
          if (gclock() - t0 > kSpinNs) {
            set_status(status, kStTimeout);
            abort = 1;
            break;
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 4; j++) v[j] = __uint_as_float((uint32_t)w[j]);
    }
    encode4(g, base, t, q, v);
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
// [1] down tiles done (fused mode) or row blocks combined; [2 + rb] down
// tiles done in row block rb.  In the fused mode (a.fused, one or two tokens)
// the next layer's gate/up tiles rebuild their input from y themselves, so a
// layer hands over after its last down tile, and h goes from gate/up to down
// as tagged words that the down tiles poll, without counter [0]; otherwise
// the last down tile of a row block combines that block into the layer output
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
  const bool fused = a.fused != 0;
  const uint32_t epoch = fused ? *a.epoch : 0u;  // tag of layer l: epoch << 7 | l

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
    // the combine weights this layer uses: the previous layer's for the fused
    // gate/up input, else this layer's for its row-block combines
    if (fused ? l > 0 : haveB) load_combine(fused ? rec - 1 : rec);
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
          if (!cta_wait_geq(prev, fused ? units_of[l - 1] * nrbB : nrbB, hd.abort, a.status)) {
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
        if (fused && l > 0) stage_comb(gA, baseA, a, H, hd.cw, hd.cpos, m.tok + t0, n);
        else stage_x<true>(gA, baseA, xin, m.tok + t0, n);
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
        tile_dots(gA, lmA, baseA, n);
        __syncthreads();
        if (threadIdx.x < gA.R * n) {
          const int t = threadIdx.x >> gA.rlog, r = threadIdx.x & (gA.R - 1);
          const size_t at = (size_t)(m.hbase + t0 + t) * I + m.row0 + r;
          if (fused)  // a missing expert still delivers (zeros), so no reader waits for it
            st_tagged(a.h_tagged + at,
                      m.blob ? silu(row_value(gA, baseA, 0, r, t)) * row_value(gA, baseA, 1, r, t) : 0.f,
                      (epoch << 7) | (uint32_t)l);
          else if (m.blob)
            a.h[at] = silu(row_value(gA, baseA, 0, r, t)) * row_value(gA, baseA, 1, r, t);
        }
      }
      // the fused mode's h carries its own tag: no counter to publish
      if (fused) __syncthreads(); else cta_arrive(&sy[0]);
    }
    // without a down phase, the next layer's first gate/up tile goes out now
    if (!haveB && nextA) {
      __syncthreads();
      issue_A(first[2 * (l + 1)]);
    }
    // ---------------- down (+ row-block combine) ----------------
    if (haveB) {
      // every gate/up tile of this layer is done (the fused mode polls its
      // tagged h instead)
      if (!fused && !cta_wait_geq(&sy[0], tilesA, hd.abort, a.status)) {
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
          if (fused) stage_h_tagged(gB, baseB, a.h_tagged, mb.tok + t0, n, (epoch << 7) | (uint32_t)l, hd.abort, a.status);
          else stage_x<false>(gB, baseB, a.h, mb.tok + t0, n);
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
          tile_dots(gB, lmB, baseB, n);
          __syncthreads();
          if (threadIdx.x < gB.R * n) {
            const int t = threadIdx.x >> gB.rlog, r = threadIdx.x & (gB.R - 1);
            a.y[(size_t)(mb.hbase + t0 + t) * H + mb.row0 + r] = mb.blob ? row_value(gB, baseB, 0, r, t) : 0.f;
          }
        }
        if (fused) {
          cta_arrive(&sy[1]);
          continue;
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
  // fused combine: CTA 0 writes the last layer's output once its down tiles are done
  if (fused && b == 0) {
    const int L = a.n_layers;
    __syncthreads();
    load_combine(a.rec + L - 1);
    if (!cta_wait_geq(a.sync + (size_t)(L - 1) * a.sync_stride + 1, units_of[L - 1] * nrbB, hd.abort, a.status)) return;
    const int per = H / 4;
    for (int i = threadIdx.x; i < a.T * per; i += kGemvThreads) {
      const int t = i / per, q = i - t * per;
      float v[4];
      combine4(a.y, hd.cw, hd.cpos, t, q, H, a.T, a.k, a.n_shared, v);
      __nv_bfloat162 b0 = __floats2bfloat162_rn(v[0], v[1]), b1 = __floats2bfloat162_rn(v[2], v[3]);
      reinterpret_cast<uint2*>(a.out + (size_t)t * H)[q] =
          make_uint2(*reinterpret_cast<uint32_t*>(&b0), *reinterpret_cast<uint32_t*>(&b1));
    }
  }
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
  route_in_cta<PER>(a.logits + (size_t)l * a.T * a.E, a.T, a.E, a.k, a.renorm, r, a.status);
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
  const Gv g = make_gv(a.H, a.I, 2);
  return launch_one(k_dec_gate_up, a, g, a.I, (a.max_units + a.n_shared) * (a.I / g.R), pdl, s);
}

cudaError_t launch_dec_down(const DecodeArgs& a, bool pdl, cudaStream_t s) {
  const Gv g = make_gv(a.I, a.H, 1);
  return launch_one(k_dec_down, a, g, a.H, (a.max_units + a.n_shared) * (a.H / g.R), pdl, s);
}

cudaError_t launch_dec_dequant(const uint8_t* blob, const BlobLayout& lay, int mat, int H, int I, float* out,
                               cudaStream_t s) {
  const int K = mat < 2 ? H : I, rows = mat < 2 ? I : H;
  const Gv g = make_gv(K, rows, 1);
  if (!gv_ok(g, rows)) return cudaErrorInvalidValue;
  const size_t smem = kTileOff + g.total;
  cudaError_t e = cudaFuncSetAttribute(k_dec_dequant, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_dec_dequant<<<rows / g.R, kGemvThreads, smem, s>>>(blob, lay, mat, H, I, out);
  return cudaGetLastError();
}

bool decode_supported(int H, int I) { return gv_ok(make_gv(H, I, 2), I) && gv_ok(make_gv(I, H, 1), H); }

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

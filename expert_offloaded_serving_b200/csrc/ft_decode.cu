// Decode path for small batches (T <= 16): fused routing + split-K FP4 GEMV.
//
//   k_dec_gate_up   every CTA routes the T tokens itself (softmax top-k +
//                   permutation, a few hundred pairs at most), takes one unit
//                   (a distinct selected expert, or the shared expert), one
//                   128-row block of Wg/Wu and one K-slice, stages that tile in
//                   shared memory with coalesced 16-byte cp.async copies from
//                   all threads, dequantises e2m1 codes with their UE8M0 scales in
//                   registers, and reduces the K-slices of a row block across
//                   the CTAs of a thread-block cluster through distributed
//                   shared memory; the owner CTA applies SwiGLU and writes fp32 h.
//   k_dec_down      same routing; one unit, one 128-row block of Wd, one
//                   K-slice of I; launched as a programmatic dependent of the
//                   gate/up kernel so its weight tile streams in while gate/up
//                   still runs; after griddepcontrol.wait it reads h, reduces
//                   its K-slices in the cluster and writes y.  The last CTA to
//                   finish a row block (an atomic counter per row block) sums
//                   w[t][j] * y over j ascending plus the shared expert and
//                   rounds once to bf16.
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

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void st_cluster_f32(const float* local_addr, uint32_t rank, float v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local_addr)), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}

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

// Dot of 32 e2m1 codes (16 bytes) with 32 activations (16 float pairs).
__device__ __forceinline__ float chunk_dot(uint4 q, const float2* xv) {
  float2 acc = make_float2(0.f, 0.f);
  const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int wv = 0; wv < 4; wv++)
#pragma unroll
    for (int b = 0; b < 4; b++) acc = ffma2(f16x2_to_f32x2(e2m1x2_to_f16x2(qs[wv] >> (8 * b))), xv[wv * 4 + b], acc);
  return acc.x + acc.y;
}

// Scale byte of row r (0..127), block b of a staged scale tile (atoms along K).
__device__ __forceinline__ uint32_t tile_scale(const uint8_t* sc, int r, int b) {
  return sc[(b >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (b & 3)];
}

// Shared-memory position of 16-byte chunk c of tile row r (row of `pieces`
// chunks, a multiple of 4): chunks are XOR-ed with the row's low bits so that
// consecutive rows reading the same logical chunk hit different 16-byte bank
// groups.  The XOR only touches bits inside an aligned group of 8 (or 4)
// chunks, so the result stays inside the row.
__device__ __forceinline__ int swz(int c, int r, int pieces) { return c ^ (r & ((pieces & 7) ? 3 : 7)); }

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Stage one 128-row tile with 16-byte asynchronous copies issued by all
// threads: code rows [row0, row0+128), bytes [kbyte0, kbyte0 + kbytes) of each
// row (row pitch `pitch`), and the scale atoms of that row block covering
// those blocks (contiguous).  Consecutive threads take consecutive 16-byte
// pieces of a row, so each warp load is coalesced.
__device__ __forceinline__ void stage_tile(uint8_t* codes_s, uint8_t* sc_s, const uint8_t* codes_g,
                                           const uint8_t* sc_g, int row0, int pitch, int kbyte0, int kbytes,
                                           int atoms_k) {
  const int pieces = kbytes / 16;
  if (kGemvThreads % pieces == 0) {
    const int p = threadIdx.x % pieces, rstep = kGemvThreads / pieces;
    const uint8_t* src = codes_g + (size_t)row0 * pitch + kbyte0 + p * 16;
    for (int r = threadIdx.x / pieces; r < kRows; r += rstep)
      cp_async16(codes_s + r * kbytes + swz(p, r, pieces) * 16, src + (size_t)r * pitch);
  } else {
    for (int i = threadIdx.x; i < kRows * pieces; i += kGemvThreads) {
      int r = i / pieces, p = i % pieces;
      cp_async16(codes_s + r * kbytes + swz(p, r, pieces) * 16, codes_g + (size_t)(row0 + r) * pitch + kbyte0 + p * 16);
    }
  }
  const int sc_bytes = (kbytes / 64) * 512;
  const uint8_t* sg = sc_g + ((size_t)(row0 >> 7) * atoms_k + kbyte0 / 64) * 512;
  for (int i = threadIdx.x; i < sc_bytes / 16; i += kGemvThreads) cp_async16(sc_s + i * 16, sg + i * 16);
}

// ---------------------------------------------------------------------------
// shared-memory plan of a CTA (dynamic smem)
// ---------------------------------------------------------------------------
struct Plan {
  int ks, lpr, cpl;   // K-slice (elements), lanes per row, chunks per lane
  int nmat;           // 2 (gate/up) or 1 (down)
  size_t codes, scales, act, part, recv, total;
};

__host__ __device__ inline Plan make_plan(int ks, int nmat, int T) {
  Plan p;
  p.ks = ks;
  int chunks = ks / 32;
  p.lpr = 16;
  while (p.lpr > 1 && chunks % p.lpr) p.lpr >>= 1;
  p.cpl = chunks / p.lpr;
  p.nmat = nmat;
  size_t off = kTileOff;
  p.codes = off;
  off += (size_t)nmat * kRows * ks / 2;
  p.scales = off;
  off += (size_t)nmat * kRows * ks / 32;
  p.act = off;
  off += (size_t)T * ks * sizeof(float);
  p.part = off;  // [tpr][row][mat][tok] unreduced partials of the threads sharing a row
  off += (size_t)(kGemvThreads / (kRows * nmat)) * kRows * nmat * T * sizeof(float);
  p.recv = off;
  off += (size_t)kRows * nmat * T * sizeof(float);
  p.total = off;
  return p;
}

// Partial dot products of the staged tile rows with the staged activations:
// part[row][mat][tok] (unreduced over K-slices).  Each thread owns one row of
// one matrix (or a contiguous share of its chunks when a row has more threads),
// so a row needs no cross-lane reduction; activations are broadcast reads.
__device__ void tile_dots(const Plan& pl, const uint8_t* codes_s, const uint8_t* sc_s, const float* act, int m, int T,
                          float* part) {
  const int rows_total = kRows * pl.nmat;
  const int tpr = kGemvThreads / rows_total;    // threads per row: 2 (gate/up) or 4 (down)
  const int chunks = pl.ks / 32, cpt = chunks / tpr;
  const int kbytes = pl.ks / 2;
  const int rr = threadIdx.x % rows_total;      // consecutive lanes -> consecutive rows
  const int sub = threadIdx.x / rows_total;
  const int mat = rr / kRows, r = rr % kRows;
  const uint8_t* cs = codes_s + (size_t)mat * kRows * kbytes + (size_t)r * kbytes;
  const uint8_t* ss = sc_s + (size_t)mat * kRows * (pl.ks / 32);
  for (int t0 = 0; t0 < m; t0 += 2) {
    const bool two = t0 + 1 < m;
    const float* a0 = act + (size_t)t0 * pl.ks;
    const float* a1 = act + (size_t)(two ? t0 + 1 : t0) * pl.ks;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 4
    for (int cc = 0; cc < cpt; cc++) {
      const int c = sub * cpt + cc;
      const uint4 q = *reinterpret_cast<const uint4*>(cs + swz(c, r, chunks) * 16);
      const float sc = ue8m0_to_f32(tile_scale(ss, r, c));
      const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
      float2 p0 = make_float2(0.f, 0.f), p1 = make_float2(0.f, 0.f);
      float2 p2 = make_float2(0.f, 0.f), p3 = make_float2(0.f, 0.f);
      const float4* x0 = reinterpret_cast<const float4*>(a0 + c * 32);
      const float4* x1 = reinterpret_cast<const float4*>(a1 + c * 32);
#pragma unroll
      for (int wv = 0; wv < 4; wv++) {
        const float4 xa = x0[2 * wv], xb = x0[2 * wv + 1];
        const float2 w0 = f16x2_to_f32x2(e2m1x2_to_f16x2(qs[wv]));
        const float2 w1 = f16x2_to_f32x2(e2m1x2_to_f16x2(qs[wv] >> 8));
        const float2 w2 = f16x2_to_f32x2(e2m1x2_to_f16x2(qs[wv] >> 16));
        const float2 w3 = f16x2_to_f32x2(e2m1x2_to_f16x2(qs[wv] >> 24));
        p0 = ffma2(w0, make_float2(xa.x, xa.y), p0);
        p1 = ffma2(w1, make_float2(xa.z, xa.w), p1);
        p0 = ffma2(w2, make_float2(xb.x, xb.y), p0);
        p1 = ffma2(w3, make_float2(xb.z, xb.w), p1);
        if (two) {
          const float4 ya = x1[2 * wv], yb = x1[2 * wv + 1];
          p2 = ffma2(w0, make_float2(ya.x, ya.y), p2);
          p3 = ffma2(w1, make_float2(ya.z, ya.w), p3);
          p2 = ffma2(w2, make_float2(yb.x, yb.y), p2);
          p3 = ffma2(w3, make_float2(yb.z, yb.w), p3);
        }
      }
      s0 = fmaf((p0.x + p0.y) + (p1.x + p1.y), sc, s0);
      s1 = fmaf((p2.x + p2.y) + (p3.x + p3.y), sc, s1);
    }
    float* pr = part + (((size_t)sub * kRows + r) * pl.nmat + mat) * T;
    pr[t0] = s0;
    if (two) pr[t0 + 1] = s1;
  }
}

// Send this CTA's partials of the rows owned by cluster rank `o` to rank o's
// receive buffer [slice][row_in_owner][mat][tok], then cluster barrier.
__device__ void cluster_exchange(const Plan& pl, const float* part, float* recv, int S, int slice, int m, int T) {
  const int rows_per_owner = kRows / S;
  const int n = kRows * pl.nmat * m;
  const int tpr = kGemvThreads / (kRows * pl.nmat);
  for (int i = threadIdx.x; i < n; i += kGemvThreads) {
    int tok = i % m;
    int mat = (i / m) % pl.nmat;
    int r = i / (m * pl.nmat);
    int owner = r / rows_per_owner;
    int rl = r % rows_per_owner;
    float v = 0.f;
    for (int sb = 0; sb < tpr; sb++) v += part[(((size_t)sb * kRows + r) * pl.nmat + mat) * T + tok];
    const float* dst = recv + (((size_t)slice * rows_per_owner + rl) * pl.nmat + mat) * T + tok;
    if (S == 1)
      *const_cast<float*>(dst) = v;
    else
      st_cluster_f32(dst, (uint32_t)owner, v);
  }
  if (S > 1)
    cluster_sync();
  else
    __syncthreads();
}

}  // namespace

// ---------------------------------------------------------------------------
// gate/up + SwiGLU
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kGemvThreads) k_dec_gate_up(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  CtaHdr& hd = *reinterpret_cast<CtaHdr*>(smem);
  const int S = a.s_gu;
  const Plan pl = make_plan(a.H / S, 2, a.T);
  uint8_t* codes_s = smem + pl.codes;
  uint8_t* sc_s = smem + pl.scales;
  float* act = reinterpret_cast<float*>(smem + pl.act);
  float* part = reinterpret_cast<float*>(smem + pl.part);
  float* recv = reinterpret_cast<float*>(smem + pl.recv);

  const int RB = a.I / kRows;
  const int slice = blockIdx.x % S;
  const int rb = (blockIdx.x / S) % RB;
  const int u = blockIdx.x / (S * RB);

  UnitInfo ui;
  if (!resolve_unit(a, a.rec, u, ui, hd.tok)) {
    pdl_trigger();
    return;  // the whole cluster (same unit) leaves together
  }
  const uint8_t* blob = a.eptr[ui.e];
  if (blob == nullptr) {
    if (threadIdx.x == 0) set_status(a.status, kStMissing);
    pdl_trigger();
    return;
  }
  const int kbytes = pl.ks / 2, pitch = a.H / 2;
  const int atoms_k = (int)(pad_up(a.H / 32, 4) / 4);
  stage_tile(codes_s, sc_s, blob + a.lay.wg, blob + a.lay.wg_sf, rb * kRows, pitch, slice * kbytes, kbytes, atoms_k);
  stage_tile(codes_s + kRows * kbytes, sc_s + kRows * (pl.ks / 32), blob + a.lay.wu, blob + a.lay.wu_sf, rb * kRows,
             pitch, slice * kbytes, kbytes, atoms_k);
  cp_async_commit();
  pdl_trigger();
  pdl_wait();  // activations come from the previous kernel when launched as a dependent
  for (int i = threadIdx.x; i < ui.m * (pl.ks / 4); i += kGemvThreads) {
    int mm = i / (pl.ks / 4), k4 = i % (pl.ks / 4);
    int t = hd.tok[mm];
    uint2 xv = *reinterpret_cast<const uint2*>(a.x + (size_t)t * a.H + slice * pl.ks + k4 * 4);
    reinterpret_cast<float4*>(act)[i] = make_float4(bf16_bits_to_f32(xv.x & 0xffff), bf16_bits_to_f32(xv.x >> 16),
                                                    bf16_bits_to_f32(xv.y & 0xffff), bf16_bits_to_f32(xv.y >> 16));
  }
  cp_async_wait_all();
  __syncthreads();
  tile_dots(pl, codes_s, sc_s, act, ui.m, a.T, part);
  __syncthreads();
  cluster_exchange(pl, part, recv, S, slice, ui.m, a.T);
  // owner rows: sum slices in order, SwiGLU, write h
  const int rows_per_owner = kRows / S;
  for (int i = threadIdx.x; i < rows_per_owner * ui.m; i += kGemvThreads) {
    int rl = i / ui.m, tok = i % ui.m;
    float gs = 0.f, us = 0.f;
    for (int s = 0; s < S; s++) {
      gs += recv[(((size_t)s * rows_per_owner + rl) * 2 + 0) * a.T + tok];
      us += recv[(((size_t)s * rows_per_owner + rl) * 2 + 1) * a.T + tok];
    }
    int row = rb * kRows + slice * rows_per_owner + rl;
    a.h[(size_t)(ui.hbase + tok) * a.I + row] = silu(gs) * us;
  }
}

// ---------------------------------------------------------------------------
// down + combine
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kGemvThreads) k_dec_down(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  CtaHdr& hd = *reinterpret_cast<CtaHdr*>(smem);
  const int S = a.s_dn;
  const Plan pl = make_plan(a.I / S, 1, a.T);
  uint8_t* codes_s = smem + pl.codes;
  uint8_t* sc_s = smem + pl.scales;
  float* act = reinterpret_cast<float*>(smem + pl.act);
  float* part = reinterpret_cast<float*>(smem + pl.part);
  float* recv = reinterpret_cast<float*>(smem + pl.recv);

  const int RB = a.H / kRows;
  const int slice = blockIdx.x % S;
  const int rb = (blockIdx.x / S) % RB;
  const int u = blockIdx.x / (S * RB);

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
  const int kbytes = pl.ks / 2, pitch = a.I / 2;
  const int atoms_k = (int)(pad_up(a.I / 32, 4) / 4);
  stage_tile(codes_s, sc_s, blob + a.lay.wd, blob + a.lay.wd_sf, rb * kRows, pitch, slice * kbytes, kbytes, atoms_k);
  cp_async_commit();
  pdl_trigger();
  pdl_wait();  // h is written by the gate/up kernel
  for (int i = threadIdx.x; i < ui.m * (pl.ks / 4); i += kGemvThreads) {
    int mm = i / (pl.ks / 4), k4 = i % (pl.ks / 4);
    reinterpret_cast<float4*>(act)[i] =
        *reinterpret_cast<const float4*>(a.h + (size_t)(ui.hbase + mm) * a.I + slice * pl.ks + k4 * 4);
  }
  cp_async_wait_all();
  __syncthreads();
  tile_dots(pl, codes_s, sc_s, act, ui.m, a.T, part);
  __syncthreads();
  cluster_exchange(pl, part, recv, S, slice, ui.m, a.T);
  const int rows_per_owner = kRows / S;
  const int row0 = rb * kRows + slice * rows_per_owner;
  for (int i = threadIdx.x; i < rows_per_owner * ui.m; i += kGemvThreads) {
    int rl = i / ui.m, tok = i % ui.m;
    float ys = 0.f;
    for (int s = 0; s < S; s++) ys += recv[((size_t)s * rows_per_owner + rl) * a.T + tok];
    a.y[(size_t)(ui.hbase + tok) * a.H + row0 + rl] = ys;
  }
  // last CTA of this row group combines
  __threadfence();
  __syncthreads();
  const int units = a.rec->n_active + a.n_shared;
  if (threadIdx.x == 0) {
    int* ctr = a.counters + rb * S + slice;
    int old = atomicAdd(ctr, 1);
    hd.last = (old == units - 1);
    if (hd.last) *ctr = 0;
  }
  __syncthreads();
  if (!hd.last) return;
  __threadfence();
  for (int i = threadIdx.x; i < a.T * rows_per_owner; i += kGemvThreads) {
    int t = i / rows_per_owner, rl = i % rows_per_owner;
    int n = row0 + rl;
    float acc = 0.f;
    for (int j = 0; j < a.k; j++) {
      int f = t * a.k + j;
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
int choose_slices(int K) {
  // largest S <= 8 with K/S a multiple of 128 in [512, 1024] (else S = 1)
  for (int s = 8; s >= 2; s--)
    if (K % (s * 128) == 0 && K / s >= 512 && K / s <= 1024) return s;
  return 1;
}

size_t decode_smem_bytes(int K, int S, int nmat, int T) { return make_plan(K / S, nmat, T).total; }

static cudaError_t launch_one(void (*kern)(DecodeArgs), const DecodeArgs& a, int grid, int cluster, size_t smem,
                              bool pdl, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute at[2];
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(kGemvThreads);
  cfg.gridDim = dim3(grid);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = cluster;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 2;
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
  const int U = a.max_units + a.n_shared;
  return launch_one(k_dec_gate_up, a, U * (a.I / kRows) * a.s_gu, a.s_gu,
                    decode_smem_bytes(a.H, a.s_gu, 2, a.T), pdl, s);
}

cudaError_t launch_dec_down(const DecodeArgs& a, bool pdl, cudaStream_t s) {
  const int U = a.max_units + a.n_shared;
  return launch_one(k_dec_down, a, U * (a.H / kRows) * a.s_dn, a.s_dn, decode_smem_bytes(a.I, a.s_dn, 1, a.T),
                    pdl, s);
}

}  // namespace ft

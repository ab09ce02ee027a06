// Dataflow decode over a stack of resident layers, for one or two tokens: one
// persistent cooperative launch in which the data itself carries every
// dependency between CTAs (no counters, no fences on the critical path).
//
// Per layer, two phases:
//   gate/up  tile = (unit, R rows of Wg and Wu) over the full hidden K.  Its
//            input is the layer's x; its output h = silu(Wg x) * (Wu x) goes
//            out as tagged 64-bit words (tag << 32 | fp32 bits).
//   down     tile = (slice of rb output rows) x (every unit of the layer).  It
//            stages the h of all units, computes y for its rows of every unit,
//            combines them (sum over j ascending of w[t][j] * y, then the
//            shared expert, one bf16 rounding) and publishes the next layer's
//            x for its rows as tagged words (tag << 32 | two bf16), or writes
//            the stack's output after the last layer.
// A reader polls exactly the words it needs until their tags name this
// launch and layer (tag = launch counter << 7 | layer); a word is stored and
// loaded whole, so the value that arrives with the tag is the value written
// with it.  Each CTA streams its next tile's weights (bulk copies for the
// codes, 4-byte cp.async for the scale words) as soon as the buffer is free,
// so weights move one phase ahead of the compute.
//
// Why the down tile spans every unit: the next layer's gate/up tiles need all
// of x, and x is the combination of every unit's y.  A tile that owns rows of
// every unit combines them itself, so each gate/up CTA reads the finished
// bf16 x (8 KB at hidden 2048) instead of every unit's fp32 y (72 KB).
//
// Arithmetic is that of the per-layer kernels (ft_decode.cu), bit for bit:
// the same re-encoding of x and h, the same chunk dot products, the same
// reduction tree over a row's lanes (pairing lanes by the same bits in the
// same order whatever the rows per step), parts added in ascending order,
// the same combine order.  So a stack equals the same layers run one
// ft_moe_layer_forward at a time.
//
// Pages: experts are computed from weights in VRAM and their partial results
// summed exactly (jansverre.net, "Hvorfor er båndbredden viktigere enn antall
// kjerner?"); a gate picks a few experts per token (aiforradalom.hu, "A
// Mixture-of-Experts (MoE) kihívásai és a FreeToken megoldásai").
#include <algorithm>

#include "ft_common.cuh"
#include "ft_decode.h"
#include "ft_tile.cuh"

namespace ft {
using namespace tile;
namespace {

constexpr int kWarpsF = kGemvThreads / 32;
constexpr int kIssuerF = 32;  // lane 0 of warp 1 issues the bulk weight copies

// One unit of a layer (a distinct routed expert or a shared expert).
struct FlowUnit {
  const uint8_t* blob;  // NULL: the expert is missing (its outputs count as zero)
  int16_t hrow;         // first h row of the unit
  int8_t m;             // tokens of the unit (1 or 2)
  int8_t tok[2];        // their token ids
  int8_t pad[3];
  float ts[3];          // NVFP4: the fp32 scales of Wg, Wu, Wd (else 1)
  int32_t pad2;
};
static_assert(sizeof(FlowUnit) == 32, "FlowUnit");

// One (token, rank) pair of a layer, for the combine.
struct FlowPair {
  float w;        // combine weight
  uint8_t unit;   // unit holding the pair's expert
  uint8_t slot;   // the pair's token slot within that unit
  uint8_t on;     // the expert's blob is present (else its y counts as zero)
  uint8_t pad;
};
static_assert(sizeof(FlowPair) == 8, "FlowPair");

struct FlowLayerHdr {
  int32_t units;    // U
  int32_t rb;       // down rows per unit per tile (even)
  int32_t nd;       // down tiles, ceil(H / rb)
  int32_t tiles_a;  // gate/up tiles, U * I / R
};

// Layer record in shared memory: header, FlowUnit[umax], FlowPair[pairs].
__host__ __device__ inline size_t flow_layer_bytes(int umax, int pairs) {
  return (sizeof(FlowLayerHdr) + (size_t)umax * sizeof(FlowUnit) + (size_t)pairs * sizeof(FlowPair) + 15) & ~(size_t)15;
}

struct FlowHdr {
  uint64_t bar[2];  // completion of the bulk weight copies into buffers A and B
  int32_t abort;
  int32_t pad[3];
};

// Down-tile geometry: the GEMV lane mapping for K = I, with rows_cap rows (all
// units) and nh activation rows staged at once.
__host__ __device__ inline Gv make_gd(int I, int rows_cap, int nh, int fmt) {
  Gv g = make_gv(I, 1 << 30, 1, fmt);
  g.R = rows_cap;
  g.rlog = 0;
  g.codes = 0;
  g.scales = (size_t)rows_cap * g.rowb;
  g.xh = g.scales + (size_t)rows_cap * g.atoms * 4;
  g.xinv = g.xh + (size_t)nh * I * (fmt == kFmtBf16 ? 4 : 2);
  g.red = g.xinv + (fmt == kFmtBf16 ? 0 : (((size_t)nh * g.chunks * 4 + 15) & ~(size_t)15));
  g.total = (g.red + (size_t)g.parts * rows_cap * kMT * 4 + 127) & ~(size_t)127;
  return g;
}

__host__ __device__ inline size_t round128(size_t v) { return (v + 127) & ~(size_t)127; }

__device__ __forceinline__ void ld_tagged2(const uint64_t* p, uint64_t& w0, uint64_t& w1) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(w0), "=l"(w1) : "l"(p) : "memory");
}
__device__ __forceinline__ void st_tagged_raw(uint64_t* p, uint64_t w) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}

// The gate/up activations of tokens toks[0 .. n) from the tagged x words of
// this layer: a word whose tag differs has not arrived and is read again, for
// at most kSpinNs (then the timeout bit and the CTA's abort flag are set).
// Re-encoded like stage_x.
__device__ __forceinline__ void stage_x_tagged(const Gv& g, uint8_t* base, const uint64_t* xt, const int8_t* toks,
                                               int n, uint32_t tag, int& abort, int* status) {
  const int per = g.K / 4;
  const int items = (n > 1 ? kMT : 1) * per;
  for (int i = threadIdx.x; i < items; i += kGemvThreads) {
    const int t = i / per, q = i - t * per;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (t < n) {
      const uint64_t* p = xt + (size_t)toks[t] * (g.K / 2) + 2 * q;
      uint64_t w0, w1;
      ld_tagged2(p, w0, w1);
      if ((uint32_t)(w0 >> 32) != tag || (uint32_t)(w1 >> 32) != tag) {
        const uint64_t t0 = gclock();
        for (uint32_t n = 1;; n++) {
          __nanosleep(20);
          ld_tagged2(p, w0, w1);
          if ((uint32_t)(w0 >> 32) == tag && (uint32_t)(w1 >> 32) == tag) break;
          if ((n & 15) == 0 && gclock() - t0 > kSpinNs) {
            set_status(status, kStTimeout);
            abort = 1;
            break;
          }
        }
      }
      v[0] = __uint_as_float((uint32_t)w0 << 16);
      v[1] = __uint_as_float((uint32_t)w0 & 0xffff0000u);
      v[2] = __uint_as_float((uint32_t)w1 << 16);
      v[3] = __uint_as_float((uint32_t)w1 & 0xffff0000u);
    }
    encode4(g, base, t, q, v);
  }
}

// The down tile's activations: every h row 0 .. nh-1 of the layer (all
// units), from the tagged h words, re-encoded like stage_x.  Each thread
// loads up to kHBatch items before it looks at any tag, so the L2 round
// trips of its items overlap.
constexpr int kHBatch = 4;
__device__ __forceinline__ void stage_h_all(const Gv& g, uint8_t* base, const uint64_t* ht, int nh, uint32_t tag,
                                            int& abort, int* status) {
  const int per = g.K / 4;
  const int items = nh * per;  // a multiple of 32: warps stay whole for encode4's shuffles
  for (int i0 = 0; i0 < items; i0 += kHBatch * kGemvThreads) {
    uint64_t w[kHBatch][4];
#pragma unroll
    for (int j = 0; j < kHBatch; j++) {
      const int i = i0 + j * kGemvThreads + threadIdx.x;
      if (i < items) ld_tagged4(ht + (size_t)(i / per) * g.K + 4 * (i % per), w[j]);
    }
#pragma unroll
    for (int j = 0; j < kHBatch; j++) {
      const int i = i0 + j * kGemvThreads + threadIdx.x;
      if (i >= items) break;
      const int t = i / per, q = i - t * per;
      auto ready = [&]() {
        return (uint32_t)(w[j][0] >> 32) == tag && (uint32_t)(w[j][1] >> 32) == tag &&
               (uint32_t)(w[j][2] >> 32) == tag && (uint32_t)(w[j][3] >> 32) == tag;
      };
      if (!ready()) {
        const uint64_t* p = ht + (size_t)t * g.K + 4 * q;
        const uint64_t t0 = gclock();
        for (uint32_t n = 1;; n++) {
          __nanosleep(20);
          ld_tagged4(p, w[j]);
          if (ready()) break;
          if ((n & 15) == 0 && gclock() - t0 > kSpinNs) {
            set_status(status, kStTimeout);
            abort = 1;
            break;
          }
        }
      }
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; e++) v[e] = __uint_as_float((uint32_t)w[j][e]);
      encode4(g, base, t, q, v);
    }
  }
}

// Partial sums of the down tile: unit u's rows u*rb .. u*rb + rb - 1 against
// the unit's h rows.  The tile's rows, unit-major, are taken two at a time
// (rb is even, so a pair never straddles units); lane group g takes the pairs
// [g*ppg, (g+1)*ppg).  Every lane of a warp runs the same number of steps, so
// the reduction's shuffles see the whole warp; pairs past the end compute
// zeros and are not stored.  NT = tokens per pass (2 when any unit has two).
template <int NT, int F>
__device__ __forceinline__ void dtile_dots(const Gv& g, const LaneMap& m, uint8_t* base, const FlowUnit* un, int U,
                                           int rb) {
  if (!m.on) return;
  const uint8_t* codes = base + g.codes;
  const uint32_t* sc = reinterpret_cast<const uint32_t*>(base + g.scales);
  float* red = reinterpret_cast<float*>(base + g.red);
  const bool cv = m.c < g.chunks;
  const int npairs = U * rb / 2;
  const int ppg = (npairs + g.groups - 1) / g.groups;
  const int lmask = (g.lpr >> 1) - 1;
  int cur = -1;
  uint32_t x[kMT][16];
  float xi[kMT] = {0.f, 0.f};
  float xf[kMT][32];
#pragma unroll
  for (int t = 0; t < kMT; t++) zero_act<F>(x[t], xi[t], xf[t]);
  for (int jp = 0; jp < ppg; jp++) {
    const int p = m.grp * ppg + jp;
    const bool pv = p < npairs;
    const int row = 2 * p;
    const int u = pv ? row / rb : cur;
    if (pv && u != cur && cv) {
      cur = u;
      const FlowUnit f = un[u];
#pragma unroll
      for (int t = 0; t < NT; t++) {
        if (t < f.m) load_act<F>(g, base, f.hrow + t, m.c, x[t], xi[t], xf[t]);
        else zero_act<F>(x[t], xi[t], xf[t]);
      }
    }
    float v[4][kMT];
#pragma unroll
    for (int uu = 0; uu < 2; uu++) {
      v[uu][0] = v[uu][1] = 0.f;
      if (cv && pv) chunk_value<NT, F>(g, codes, sc, row + uu, m.c, x, xi, xf, v[uu]);
    }
    const int sel = group_reduce<2, NT>(v, g.lpr);
    if (pv && ((threadIdx.x & 31) & lmask) == 0) {
      float* o = red + ((size_t)m.part * g.R + row + sel) * kMT;
#pragma unroll
      for (int t = 0; t < NT; t++) o[t] = v[0][t];
    }
  }
}

// y of tile row `row` (unit-major) for token slot t: the parts in ascending order.
__device__ __forceinline__ float dtile_y(const Gv& g, const uint8_t* base, int row, int t) {
  const float* red = reinterpret_cast<const float*>(base + g.red);
  float s = red[(size_t)row * kMT + t];
  for (int p = 1; p < g.parts; p++) s += red[((size_t)p * g.R + row) * kMT + t];
  return s;
}

}  // namespace

// See the file comment.  HS, IS: hidden and intermediate size fixed at compile
// time (the tile geometry then folds to constants), or 0, 0 for any shape.
// TT: 1 for a build that takes one token only (its dot-product loops are
// the one-token ones), 0 for one or two tokens.  RUG: rows per step of the
// gate/up tile fixed at compile time (the shape-specific builds), or 0.
template <int HS, int IS, int F, int TT, int RUG>
__global__ void __launch_bounds__(kGemvThreads, 1) k_dec_flow(FlowArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int H = HS ? HS : a.H, I = IS ? IS : a.I;
  const int T = TT ? TT : a.T, k = a.k, S = a.n_shared, P = T * k, NH = P + S * T;
  const int umax = min(a.E, P) + S;
  const Gv gA = make_gv(H, I, 2, F);
  const Gv gB = make_gd(I, a.rows_cap, NH, F);
  uint8_t* baseA = smem;
  uint8_t* baseB = smem + round128(gA.total);
  FlowHdr& hd = *reinterpret_cast<FlowHdr*>(baseB + gB.total);
  uint8_t* ltab = reinterpret_cast<uint8_t*>(&hd + 1);
  const size_t lstride = flow_layer_bytes(umax, P);
  const LaneMap lmA = lane_map(gA), lmB = lane_map(gB);
  const int G = gridDim.x, b = blockIdx.x;
  const int nrbA = I / gA.R;
  const uint32_t epoch = *a.epoch;
  auto lhdr = [&](int l) -> const FlowLayerHdr& { return *reinterpret_cast<const FlowLayerHdr*>(ltab + l * lstride); };
  auto lunits = [&](int l) { return reinterpret_cast<const FlowUnit*>(ltab + l * lstride + sizeof(FlowLayerHdr)); };
  auto lpairs = [&](int l) {
    return reinterpret_cast<const FlowPair*>(ltab + l * lstride + sizeof(FlowLayerHdr) + umax * sizeof(FlowUnit));
  };

  // ---- prologue: warp w resolves layers w, w + 16, ... into shared memory ----
  if (threadIdx.x == 0) {
    hd.abort = 0;
    mbar_init(&hd.bar[0]);
    mbar_init(&hd.bar[1]);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  {
    const int lane = threadIdx.x & 31;
    // down rows per unit: about H / G rows per tile (one tile per CTA), at most
    // rows_cap over all units
    const int rb_g = 2 * ((H + 2 * G - 1) / (2 * G));
    for (int l = threadIdx.x >> 5; l < a.n_layers; l += kWarpsF) {
      const Route* rec = a.rec + l;
      const uint8_t* const* eptr = a.eptr + (size_t)l * a.n_blobs;
      uint8_t* L = ltab + l * lstride;
      FlowUnit* un = reinterpret_cast<FlowUnit*>(L + sizeof(FlowLayerHdr));
      FlowPair* pr = reinterpret_cast<FlowPair*>(L + sizeof(FlowLayerHdr) + umax * sizeof(FlowUnit));
      const int na = rec->n_active, U = na + S;
      for (int u = lane; u < U; u += 32) {
        FlowUnit f;
        int e;
        if (u < na) {
          e = rec->unit_e[u];
          const int p0 = rec->unit_p0[u];
          f.m = (int8_t)rec->unit_m[u];
          f.hrow = (int16_t)p0;
          for (int t = 0; t < 2; t++) f.tok[t] = (int8_t)(t < f.m ? rec->perm[p0 + t] / k : 0);
        } else {
          e = a.E + (u - na);
          f.m = (int8_t)T;
          f.hrow = (int16_t)(P + (u - na) * T);
          f.tok[0] = 0;
          f.tok[1] = 1;
        }
        f.blob = eptr[e];
        f.pad[0] = f.pad[1] = f.pad[2] = 0;
        f.pad2 = 0;
        for (int q = 0; q < 3; q++)
          f.ts[q] = (F == kFmtNv && f.blob) ? reinterpret_cast<const float*>(f.blob + a.lay.ts)[q] : 1.f;
        if (!f.blob) set_status(a.status, kStMissing);
        un[u] = f;
      }
      for (int f = lane; f < P; f += 32) {
        const int pos = rec->pos[f];
        int u = 0;  // the routed units' first positions ascend
        while (u + 1 < na && rec->unit_p0[u + 1] <= pos) u++;
        FlowPair q;
        q.w = rec->w[f];
        q.unit = (uint8_t)u;
        q.slot = (uint8_t)(pos - rec->unit_p0[u]);
        q.on = eptr[rec->unit_e[u]] != nullptr;
        q.pad = 0;
        pr[f] = q;
      }
      if (lane == 0) {
        FlowLayerHdr h;
        h.units = U;
        h.rb = max(2, min(rb_g, 2 * (a.rows_cap / (2 * U))));
        h.nd = (H + h.rb - 1) / h.rb;
        h.tiles_a = U * nrbA;
        *reinterpret_cast<FlowLayerHdr*>(L) = h;
      }
    }
  }
  __syncthreads();

  // ---- weight streaming ----
  uint32_t phase[2] = {0u, 0u};      // parity of each buffer's next mbarrier phase
  bool pending[2] = {false, false};  // bulk copies issued into the buffer and not waited for
  // cp.async groups (scale words) are committed in issue order; `seq` numbers
  // them so that a wait can leave a newer group of the other buffer in flight
  int seq = 0, seqbuf[2] = {-1, -1};
  auto issue_A = [&](int l, int i) {
    const FlowUnit f = lunits(l)[i / nrbA];
    const int row0 = (i % nrbA) * gA.R;
    if (threadIdx.x == kIssuerF) {
      const uint32_t bytes = (uint32_t)gA.R * (uint32_t)gA.rowb;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_expect_tx(&hd.bar[0], f.blob ? 2u * bytes : 0u);
      if (f.blob) {
        bulk_g2s(baseA + gA.codes, f.blob + a.lay.wg + (size_t)row0 * gA.rowb, bytes, &hd.bar[0]);
        bulk_g2s(baseA + gA.codes + bytes, f.blob + a.lay.wu + (size_t)row0 * gA.rowb, bytes, &hd.bar[0]);
      }
    }
    if (f.blob) {
      stage_scales(gA, baseA, 0, f.blob + a.lay.wg_sf, row0);
      stage_scales(gA, baseA, 1, f.blob + a.lay.wu_sf, row0);
    }
    cp_async_commit();
    seqbuf[0] = seq++;
    pending[0] = true;
  };
  auto issue_B = [&](int l, int d) {
    const FlowLayerHdr lh = lhdr(l);
    const FlowUnit* un = lunits(l);
    const int rb = lh.rb, n0 = d * rb, nv = min(rb, H - n0);
    const uint32_t rbytes = (uint32_t)nv * (uint32_t)gB.rowb;
    if (threadIdx.x == kIssuerF) {
      uint32_t total = 0;
      for (int u = 0; u < lh.units; u++)
        if (un[u].blob) total += rbytes;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_expect_tx(&hd.bar[1], total);
      for (int u = 0; u < lh.units; u++)
        if (un[u].blob)
          bulk_g2s(baseB + gB.codes + (size_t)u * rb * gB.rowb, un[u].blob + a.lay.wd + (size_t)n0 * gB.rowb, rbytes,
                   &hd.bar[1]);
    }
    uint32_t* sd = reinterpret_cast<uint32_t*>(baseB + gB.scales);
    const int per_u = nv * gB.atoms;  // 0 for BF16: no scales
    for (int i = threadIdx.x; i < lh.units * per_u; i += kGemvThreads) {
      const int u = i / per_u, j = i - u * per_u, r = j / gB.atoms, at = j - r * gB.atoms;
      const uint8_t* bl = un[u].blob;
      if (bl) cp_async4(sd + (size_t)(u * rb + r) * gB.atoms + at, bl + a.lay.wd_sf + sf_word(n0 + r, at, gB.atoms));
    }
    cp_async_commit();
    seqbuf[1] = seq++;
    pending[1] = true;
  };
  // every thread waits for buffer buf: its scale words, then its codes
  auto wait_buf = [&](int buf) {
    if (seqbuf[1 - buf] > seqbuf[buf] && pending[1 - buf]) asm volatile("cp.async.wait_group 1;" ::: "memory");
    else cp_async_wait_all();
    if (!mbar_wait(&hd.bar[buf], phase[buf], a.status)) hd.abort = 1;
    phase[buf] ^= 1u;
    pending[buf] = false;
  };
  auto drain = [&]() {
    for (int buf = 0; buf < 2; buf++)
      if (pending[buf]) mbar_wait(&hd.bar[buf], phase[buf], a.status);
    cp_async_wait_all();
  };

  if (b < lhdr(0).tiles_a) issue_A(0, b);
  if (b < lhdr(0).nd) issue_B(0, b);

  uint64_t* tl = nullptr;  // this CTA's stamps of the current layer (timeline attached)
  auto stamp = [&](int i) {
    if (tl && threadIdx.x == 0) tl[i] = gclock();
  };
  for (int l = 0; l < a.n_layers; l++) {
    const FlowLayerHdr lh = lhdr(l);
    const FlowUnit* un = lunits(l);
    const uint32_t tag = (epoch << 7) | (uint32_t)l;
    const bool last = l + 1 == a.n_layers;
    tl = a.timeline ? a.timeline + ((size_t)l * G + b) * 8 : nullptr;
    stamp(0);
    // ---------------- gate/up + SwiGLU ----------------
    for (int i = b; i < lh.tiles_a; i += G) {
      if (i != b) issue_A(l, i);  // buffer A is free since the previous tile's compute
      const FlowUnit f = un[i / nrbA];
      const int row0 = (i % nrbA) * gA.R;
      __syncthreads();
      if (l == 0) {
        const int toks[2] = {f.tok[0], f.tok[1]};
        stage_x<true>(gA, baseA, a.x0, toks, f.m);
      } else {
        stage_x_tagged(gA, baseA, a.x_tagged, f.tok, f.m, tag, hd.abort, a.status);
      }
      wait_buf(0);
      __syncthreads();
      if (hd.abort) {
        drain();
        return;
      }
      if (i == b) stamp(1);
      tile_dots<F, TT, RUG>(gA, lmA, baseA, f.m);
      __syncthreads();
      if (i == b) stamp(7);
      if (threadIdx.x < gA.R * f.m) {
        const int t = threadIdx.x >> gA.rlog, r = threadIdx.x & (gA.R - 1);
        float gv = row_value(gA, baseA, 0, r, t), uv = row_value(gA, baseA, 1, r, t);
        if (F == kFmtNv) {
          gv *= f.ts[0];
          uv *= f.ts[1];
        }
        // a missing expert still delivers (zeros), so no reader waits for it
        st_tagged(a.h_tagged + (size_t)(f.hrow + t) * I + row0 + r, f.blob ? silu(gv) * uv : 0.f, tag);
      }
      __syncthreads();
    }
    if (b < lh.tiles_a) stamp(2);
    // buffer A is free: the next layer's first gate/up tile streams in now
    if (!last && b < lhdr(l + 1).tiles_a) issue_A(l + 1, b);
    // ---------------- down + combine, over every unit ----------------
    if (b < lh.nd) {
      stage_h_all(gB, baseB, a.h_tagged, NH, tag, hd.abort, a.status);
      const FlowPair* pr = lpairs(l);
      const int rb = lh.rb, na = lh.units - S;
      for (int d = b; d < lh.nd; d += G) {
        if (d != b) issue_B(l, d);
        wait_buf(1);
        __syncthreads();
        if (hd.abort) {
          drain();
          return;
        }
        if (d == b) stamp(3);
        if (TT != 1 && T > 1) dtile_dots<2, F>(gB, lmB, baseB, un, lh.units, rb);
        else dtile_dots<1, F>(gB, lmB, baseB, un, lh.units, rb);
        __syncthreads();
        if (d == b) stamp(5);
        const int n0 = d * rb, nv = min(rb, H - n0), half = nv / 2;
        // warp w combines output pairs w, w + 16, ...: lane j < k loads routed
        // pair j's two y values, lane k + s the shared expert s's; the sum is
        // taken in the fixed order (routed pairs ascending by fused
        // multiply-add, then the shared experts) from the lanes' values
        const int lane = threadIdx.x & 31;
        for (int i = threadIdx.x >> 5; i < T * half; i += kWarpsF) {
          const int t = i / half, nl = 2 * (i - t * half);
          float w = 0.f, y0 = 0.f, y1 = 0.f;
          if (lane < k) {
            const FlowPair q = pr[t * k + lane];
            w = q.w;
            if (q.on) {
              const float ts = F == kFmtNv ? un[q.unit].ts[2] : 1.f;
              y0 = dtile_y(gB, baseB, q.unit * rb + nl, q.slot);
              y1 = dtile_y(gB, baseB, q.unit * rb + nl + 1, q.slot);
              if (F == kFmtNv) {
                y0 *= ts;
                y1 *= ts;
              }
            }
          } else if (lane < k + S) {
            const int u = na + (lane - k);
            if (un[u].blob) {
              const float ts = F == kFmtNv ? un[u].ts[2] : 1.f;
              y0 = dtile_y(gB, baseB, u * rb + nl, t);
              y1 = dtile_y(gB, baseB, u * rb + nl + 1, t);
              if (F == kFmtNv) {
                y0 *= ts;
                y1 *= ts;
              }
            }
          }
          float o[2] = {0.f, 0.f};
          for (int j = 0; j < k; j++) {
            const float wj = __shfl_sync(0xffffffffu, w, j);
            o[0] = fmaf(wj, __shfl_sync(0xffffffffu, y0, j), o[0]);
            o[1] = fmaf(wj, __shfl_sync(0xffffffffu, y1, j), o[1]);
          }
          for (int s2 = 0; s2 < S; s2++) {
            o[0] += __shfl_sync(0xffffffffu, y0, k + s2);
            o[1] += __shfl_sync(0xffffffffu, y1, k + s2);
          }
          if (lane != 0) continue;
          __nv_bfloat162 bb = __floats2bfloat162_rn(o[0], o[1]);
          const uint32_t pairbits = *reinterpret_cast<uint32_t*>(&bb);
          const size_t at = (size_t)t * H + n0 + nl;
          if (last) reinterpret_cast<uint32_t*>(a.out)[at / 2] = pairbits;
          else st_tagged_raw(a.x_tagged + at / 2, ((uint64_t)((epoch << 7) | (uint32_t)(l + 1)) << 32) | pairbits);
        }
        if (d == b) stamp(6);
        __syncthreads();
      }
    }
    if (b < lh.nd) stamp(4);
    // buffer B is free: the next layer's first down tile streams in now
    if (!last && b < lhdr(l + 1).nd) issue_B(l + 1, b);
  }
  drain();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
FlowGeom flow_geometry(int H, int I, int T, int k, int S, int E, int n_layers, int fmt) {
  FlowGeom fg{};
  if (T < 1 || T > 2 || n_layers < 1 || n_layers > 127) return fg;
  const Gv gA = make_gv(H, I, 2, fmt);
  if (!gv_ok(gA, I)) return fg;
  const Gv l = make_gv(I, 1 << 30, 1, fmt);
  if (l.rsets <= 0 || I % 128) return fg;
  const int P = T * k, NH = P + S * T, umax = std::min(E, P) + S;
  if (umax > 255) return fg;
  // down-tile rows over all units: up to 256, and about 64 KB of codes
  int rows_cap = std::min(256, (int)(65536 / l.rowb));
  rows_cap &= ~1;
  if (rows_cap < 2 * umax) rows_cap = 2 * umax;
  const Gv gB = make_gd(I, rows_cap, NH, fmt);
  const size_t smem = round128(gA.total) + gB.total + sizeof(FlowHdr) + (size_t)n_layers * flow_layer_bytes(umax, P);
  fg.rows_cap = rows_cap;
  fg.smem = smem;
  fg.ok = smem <= 227 * 1024;
  return fg;
}

cudaError_t launch_dec_flow(const FlowArgs& a, cudaStream_t s) {
  const int F = a.lay.fmt;
  const FlowGeom fg = flow_geometry(a.H, a.I, a.T, a.k, a.n_shared, a.E, a.n_layers, F);
  if (!fg.ok || a.rows_cap != fg.rows_cap) return cudaErrorInvalidValue;
  // the 35B-class shape (hidden 2048, intermediate 512) has its own builds;
  // MXFP4 at one token also a build with only the one-token loops, whose
  // gate/up tile (32 rows of each matrix, 8 lane groups) takes 4 rows of
  // each matrix in one step
  const bool s35 = a.H == 2048 && a.I == 512;
  void (*kern)(FlowArgs) =
      F == kFmtNv     ? (s35 ? k_dec_flow<2048, 512, kFmtNv, 0, 0> : k_dec_flow<0, 0, kFmtNv, 0, 0>)
      : F == kFmtBf16 ? (s35 ? k_dec_flow<2048, 512, kFmtBf16, 0, 0> : k_dec_flow<0, 0, kFmtBf16, 0, 0>)
      : s35           ? (a.T == 1 ? k_dec_flow<2048, 512, kFmtMx, 1, 8> : k_dec_flow<2048, 512, kFmtMx, 0, 0>)
                      : k_dec_flow<0, 0, kFmtMx, 0, 0>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fg.smem);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0, occ = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
      (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGemvThreads, fg.smem)) != cudaSuccess)
    return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(kGemvThreads);
  cfg.gridDim = dim3(nsm);  // one CTA per SM: every CTA waits on others, all must be resident
  cfg.dynamicSmemBytes = fg.smem;
  cfg.stream = s;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace ft

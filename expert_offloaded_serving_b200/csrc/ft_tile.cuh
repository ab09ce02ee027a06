// GEMV tile of the decode kernels and the synchronisation primitives of the
// persistent decode kernels: shared by ft_decode.cu (routing, per-layer
// kernels, counter-synchronised stack) and ft_decode_flow.cu (the dataflow
// stack).  sm_100a only; device code, all inline.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "ft_common.cuh"

namespace ft {
namespace tile {

constexpr int kGemvThreads = 512;   // threads of every GEMV CTA

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

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
// consecutive weight rows of nmat matrices over the full K of one unit, for
// up to kMT tokens per pass.
//
// MXFP4 and NVFP4 weights: the legacy tensor cores (mma.sync m16n8k16, f16
// operands, fp32 accumulate).  The activations of a pass are first
// re-encoded in shared memory as f16 with one power-of-two factor per
// 32-element block, chosen so that the block's largest magnitude lands in
// [2^14, 2^15): a bf16 x is re-encoded exactly (down to 2^-28 of its block's
// largest element), an fp32 h is rounded to 11 significant bits.  A weight
// code becomes f16 exactly (cvt.rn.f16x2.e2m1x2) and each product w*x is exact
// in fp32.  The work is cut into tasks of 16 rows x one K part (8 blocks of
// 32, or 4 when K is not a multiple of 256); a warp takes tasks in turn.  In
// a task the 8 columns of the MMA are (block, token) pairs: the activation
// operand is block-diagonal (column n holds only block n's activations, at
// the two K positions the column owns in each instruction), so 16
// instructions, each taking elements 2i, 2i+1 of every block, leave in
// column n the dot product of the 16 rows with block n alone.  Each block's
// value is then that dot times (weight scale x inverse activation factor)
// (NVFP4: the two 16-element halves accumulate apart, each times its E4M3
// scale); a row's part sum adds its blocks' values in a fixed order (a lane's
// two columns, then xor shuffles over the four lanes of a row), and a row's
// value is the sum of its parts in ascending order.  The matrix scale of
// NVFP4 multiplies a row's value once, after the reduction (by the caller).
//
// BF16 weights: CUDA cores.  K is cut into chunks of 32 weights (64 bytes);
// a lane owns one chunk, holding that chunk's fp32 activations of up to kMT
// tokens in registers, and takes the chunk in every row given to its lane
// group.  A lane group is lpr lanes (a power of two) on lpr consecutive
// chunks; rpw = 32/lpr groups share a warp; when K has more than 32 chunks,
// `parts` groups side by side cover it (warp w takes part w % parts).  Each
// weight widens to fp32 exactly and the products are summed by packed fp32
// fused multiply-adds (fma.rn.f32x2) into two accumulators; the lanes of a
// group add their chunks with xor shuffles, then the parts are added in
// ascending order through shared memory.  The activations stay fp32 (x and
// h enter exactly).
//
// Shared memory, from the tile's base:
//   codes  [nmat][R] rows of rstride bytes: a row's codes as in global memory
//          (rowb = K/2, or 2K for BF16), then padding (MXFP4/NVFP4: 64 bytes
//          when rowb is a multiple of 128, so that consecutive rows start 64
//          bytes apart modulo 128 and the 16-byte loads of a task's 8 rows
//          fall in distinct banks)
//   scales [nmat][R] rows of sstride words of four scale bytes (K/128 words
//          for MXFP4, K/64 for NVFP4, none for BF16), padded to an odd count
//   xh     MXFP4/NVFP4: [kMT] rows of xstride bytes, f16 in K order;
//          BF16: [kMT][8][K/32] x 16 B of fp32, quad i of chunk c at [t][i][c]
//   xinv   [kMT][K/32]           inverse block factors (not for BF16)
//   red    [parts][nmat][R][kMT] partial sums
// ---------------------------------------------------------------------------
constexpr int kMT = 2;                      // tokens per pass over the tile
constexpr int kWarps = kGemvThreads / 32;
constexpr size_t kSmemLimit = 220 * 1024;
constexpr size_t kTileBytes = 64 * 1024;    // weight codes per tile, about
constexpr int kRowPad = 64;                 // padding of a staged code row (MXFP4, NVFP4)

struct Gv {
  int K, chunks, atoms;
  int lpr, rpw, parts, rsets, groups;  // BF16 lane map; MXFP4/NVFP4: parts = K parts of the MMA tasks
  int R, rlog, nmat;  // rows per tile, a power of two (R = 1 << rlog)
  int fmt, rowb;      // weight format, bytes of a row's codes
  int rstride;        // bytes per staged code row
  int sstride;        // scale words per staged row
  int xstride;        // bytes per staged activation row (MXFP4, NVFP4)
  int pblk;           // blocks of 32 per K part (MXFP4, NVFP4)
  size_t codes, scales, xh, xinv, red, total;
};

// Strides of a staged tile for K and the format (rows and regions are laid
// out by the callers).
__host__ __device__ inline void gv_strides(Gv& g) {
  const bool tc = g.fmt != kFmtBf16;
  // MXFP4/NVFP4: consecutive staged rows start 64 bytes apart modulo 128, so
  // the 16-byte loads of a task's rows fall in distinct banks
  g.rstride = g.rowb + ((tc && g.rowb % 128 == 0) ? kRowPad : 0);
  g.sstride = g.atoms == 0 ? 0 : (g.atoms | 1);
  g.xstride = tc ? 2 * g.K + 16 : 0;
  g.pblk = tc ? ((g.K % 256) == 0 ? 8 : 4) : 0;
}

__host__ __device__ inline Gv make_gv(int K, int rows, int nmat, int fmt = kFmtMx, size_t tile_bytes = kTileBytes) {
  Gv g;
  g.K = K;
  g.nmat = nmat;
  g.fmt = fmt;
  g.rowb = fmt == kFmtBf16 ? 2 * K : K / 2;
  g.chunks = K / 32;
  g.atoms = fmt == kFmtMx ? K / 128 : fmt == kFmtNv ? K / 64 : 0;
  gv_strides(g);
  if (fmt == kFmtBf16) {
    g.lpr = 1;
    while (g.lpr < 32 && g.lpr < g.chunks) g.lpr <<= 1;
    g.rpw = 32 / g.lpr;
    g.parts = (g.chunks + g.lpr - 1) / g.lpr;
    g.rsets = kWarps / g.parts;  // 0 for K > 16384: not supported
    g.groups = g.rsets * g.rpw;
  } else {
    g.lpr = g.rpw = g.groups = 0;
    g.rsets = 1;
    g.parts = g.chunks / g.pblk;
  }
  // a task takes 16 rows: at least 16 rows of one matrix, or 8 of two
  const int rmin = fmt == kFmtBf16 ? 2 : (nmat == 1 ? 16 : 8);
  int R = 128;
  while (R > rmin && (size_t)R * nmat * g.rowb > tile_bytes) R >>= 1;
  if (R > rows) R = rows;
  for (;;) {
    g.codes = 0;
    g.scales = (size_t)nmat * R * g.rstride;
    g.xh = g.scales + (size_t)nmat * R * g.sstride * 4;
    g.xinv = g.xh + (fmt == kFmtBf16 ? (size_t)kMT * K * 4 : (size_t)kMT * g.xstride);
    g.red = g.xinv + (fmt == kFmtBf16 ? 0 : (((size_t)kMT * g.chunks * 4 + 15) & ~(size_t)15));
    g.total = g.red + (size_t)g.parts * nmat * R * kMT * 4;
    if (g.total <= kSmemLimit || R <= rmin) break;
    R >>= 1;
  }
  g.R = R;
  g.rlog = 0;
  while ((1 << g.rlog) < R) g.rlog++;
  return g;
}

// Shapes the decode kernels take: K and rows multiples of 128, K <= 16384,
// and (MXFP4, NVFP4) whole 16-row tasks.
__host__ __device__ inline bool gv_ok(const Gv& g, int rows) {
  return g.rsets > 0 && g.total <= kSmemLimit && rows % g.R == 0 &&
         (g.fmt == kFmtBf16 || (g.nmat * g.R) % 16 == 0);
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
  if (g.atoms == 0) return;  // BF16: no scales
  uint32_t* sd = reinterpret_cast<uint32_t*>(base + g.scales) + (size_t)mat * g.R * g.sstride;
  for (int i = threadIdx.x; i < g.R * g.atoms; i += kGemvThreads) {
    const int r = i / g.atoms, at = i - r * g.atoms;
    cp_async4(sd + (size_t)r * g.sstride + at, sc_g + sf_word(row0 + r, at, g.atoms));
  }
}

// Stage rows [row0, row0 + R) of matrix `mat` (codes at codes_g, row pitch
// rowb; scale region sc_g) into the tile with cp.async.
__device__ __forceinline__ void stage_mat(const Gv& g, uint8_t* base, int mat, const uint8_t* codes_g,
                                          const uint8_t* sc_g, int row0) {
  uint8_t* dst = base + g.codes + (size_t)mat * g.R * g.rstride;
  const uint8_t* src = codes_g + (size_t)row0 * g.rowb;
  const int per = g.rowb / 16;
  for (int i = threadIdx.x; i < g.R * per; i += kGemvThreads) {
    const int r = i / per, c = i - r * per;
    cp_async16(dst + (size_t)r * g.rstride + c * 16, src + (size_t)i * 16);
  }
  stage_scales(g, base, mat, sc_g, row0);
}

// Bulk copies of n code rows of rowb bytes from src (row pitch rowb) into the
// staged rows at dst (pitch rstride), issued by the 32 lanes of one warp and
// completing on bar.  The caller has armed bar with the bytes (lane 0) and
// synchronised the warp before.
__device__ __forceinline__ void bulk_rows_warp(const Gv& g, uint8_t* dst, const uint8_t* src, int n, uint64_t* bar);

// BF16 weights: 4 consecutive fp32 activations (group q of token t) stored as
// they are; quad i of chunk c sits at [t][i][c], 8 quads a chunk.
__device__ __forceinline__ void store4f(const Gv& g, uint8_t* base, int t, int q, const float (&v)[4]) {
  float4* xf = reinterpret_cast<float4*>(base + g.xh);
  const int c = q >> 3, i = q & 7;
  xf[((size_t)t * 8 + i) * g.chunks + c] = make_float4(v[0], v[1], v[2], v[3]);
}

// Encode 4 consecutive activations v (group q of token t) into the tile's f16
// activations; the 8 lanes of a 32-element block agree on its factor by
// shuffles, so all 32 lanes of the warp must call this together.  (BF16
// weights: stored as fp32, see store4f.)
__device__ __forceinline__ void encode4(const Gv& g, uint8_t* base, int t, int q, const float (&v)[4]) {
  if (g.fmt == kFmtBf16) {
    store4f(g, base, t, q, v);
    return;
  }
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
  // elements 4q .. 4q+3 of the token's row, in K order
  *reinterpret_cast<uint2*>(base + g.xh + (size_t)t * g.xstride + (size_t)q * 8) =
      make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
  const int c = q >> 3;
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

// Codes (16 bytes, 32 e2m1 values) and decoded UE8M0 scale of chunk c of
// staged row `row` (rows of all matrices of the tile counted in order).
__device__ __forceinline__ void tile_chunk(const Gv& g, const uint8_t* codes, const uint32_t* sc, int row, int c,
                                           uint4& q, float& s) {
  q = *reinterpret_cast<const uint4*>(codes + (size_t)row * g.rstride + c * 16);
  const uint32_t sw = sc[(size_t)row * g.sstride + (c >> 2)];
  s = ue8m0_to_f32((sw >> (8 * (c & 3))) & 0xffu);
}

// NVFP4: the codes of chunk c and the E4M3 scales of its two 16-element
// halves (adjacent bytes of one scale word: blocks 2c and 2c + 1).
__device__ __forceinline__ void tile_chunk_nv(const Gv& g, const uint8_t* codes, const uint32_t* sc, int row, int c,
                                              uint4& q, float& s0, float& s1) {
  q = *reinterpret_cast<const uint4*>(codes + (size_t)row * g.rstride + c * 16);
  const uint32_t sw = sc[(size_t)row * g.sstride + (c >> 1)] >> (16 * (c & 1));
  s0 = e4m3_to_f32(sw & 0xffu);
  s1 = e4m3_to_f32((sw >> 8) & 0xffu);
}

// BF16: the 32 weights (64 bytes) of chunk c of staged row `row`.
__device__ __forceinline__ void tile_chunk_bf16(const Gv& g, const uint8_t* codes, int row, int c, uint4 (&q)[4]) {
  const uint4* p = reinterpret_cast<const uint4*>(codes + (size_t)row * g.rstride + c * 64);
#pragma unroll
  for (int i = 0; i < 4; i++) q[i] = p[i];
}

// BF16: the dot of a chunk's 32 weights with NT tokens' fp32 activations
// xf[t][0..31]: each bf16 widens exactly to fp32, pairs meet their
// activations in packed fp32 fused multiply-adds (two accumulator lanes).
template <int NT>
__device__ __forceinline__ void chunk_dot_bf16(const uint4 (&q)[4], const float (&xf)[kMT][32], float* d) {
  float2 acc[NT];
#pragma unroll
  for (int t = 0; t < NT; t++) acc[t] = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const uint32_t ws[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const float2 w = make_float2(__uint_as_float(ws[j] << 16), __uint_as_float(ws[j] & 0xffff0000u));
      const int e = 8 * i + 2 * j;
#pragma unroll
      for (int t = 0; t < NT; t++) acc[t] = ffma2(w, make_float2(xf[t][e], xf[t][e + 1]), acc[t]);
    }
  }
#pragma unroll
  for (int t = 0; t < NT; t++) d[t] = acc[t].x + acc[t].y;
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

// BF16: the fp32 activations of staged row srow, chunk c, into registers.
__device__ __forceinline__ void load_act_bf16(const Gv& g, const uint8_t* base, int srow, int c, float (&xf)[32]) {
  const float4* p = reinterpret_cast<const float4*>(base + g.xh);
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const float4 f = p[((size_t)srow * 8 + i) * g.chunks + c];
    xf[4 * i] = f.x;
    xf[4 * i + 1] = f.y;
    xf[4 * i + 2] = f.z;
    xf[4 * i + 3] = f.w;
  }
}

__device__ __forceinline__ void zero_act_bf16(float (&xf)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i++) xf[i] = 0.f;
}

// BF16: partial sums of the staged tile's rows for NT tokens into red.  Lane
// group grp takes rows grp + j*groups, RU of them at a time.
template <int RU, int NT>
__device__ __forceinline__ void tile_dots_t(const Gv& g, const LaneMap& m, uint8_t* base, const float (&xf)[kMT][32]) {
  const uint8_t* codes = base + g.codes;
  float* red = reinterpret_cast<float*>(base + g.red);
  const bool cv = m.c < g.chunks;
  const int lmask = RU == 2 ? (g.lpr >> 1) - 1 : g.lpr - 1;
  for (int mat = 0; mat < g.nmat; mat++) {
    // the trip count is the same for every lane of a warp, so the shuffles
    // see the whole warp
    for (int j0 = 0; m.grp + j0 * g.groups < g.R; j0 += RU) {
      float v[4][kMT];
#pragma unroll
      for (int u = 0; u < RU; u++) {
        v[u][0] = v[u][1] = 0.f;
        if (cv) {
          uint4 q[4];
          tile_chunk_bf16(g, codes, mat * g.R + m.grp + (j0 + u) * g.groups, m.c, q);
          chunk_dot_bf16<NT>(q, xf, v[u]);
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

// ---------------------------------------------------------------------------
// tensor-core dot products (MXFP4, NVFP4)
// ---------------------------------------------------------------------------
// d += A (16 x 16, f16, row) x B (16 x 8, f16, col), fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Codes of elements 2i, 2i+1 of a 32-element block (byte i of its 16 bytes)
// as an f16 pair, element 2i in the low half.
template <int I>
__device__ __forceinline__ uint32_t code_pair(const uint4& q) {
  const uint32_t w = I < 4 ? q.x : I < 8 ? q.y : I < 12 ? q.z : q.w;
  return e2m1x2_to_f16x2(w >> (8 * (I & 3)));
}

// The 16 f16 pairs of block `blk` of staged activation row `row` (or zeros).
__device__ __forceinline__ void load_xblock(const Gv& g, const uint8_t* base, bool on, int row, int blk,
                                            uint32_t (&x)[16]) {
  if (on) {
    const uint4* p = reinterpret_cast<const uint4*>(base + g.xh + (size_t)row * g.xstride + (size_t)blk * 64);
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const uint4 u = p[i];
      x[4 * i] = u.x;
      x[4 * i + 1] = u.y;
      x[4 * i + 2] = u.z;
      x[4 * i + 3] = u.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; i++) x[i] = 0u;
  }
}

// One task: staged code rows r0 .. r0+15 over K part p, for NT (1 or 2)
// token columns whose activations are staged rows xrow .. xrow+n-1 (n <= NT).
// The 8 MMA columns are (block, token) pairs: column c is block c / NT of
// the group and token c % NT.  Lane (gi, ti) = (lane / 4, lane % 4) feeds the
// weight operand with the blocks of columns ti and ti + 4 (rows gi, gi + 8)
// and, when gi == ti or gi == ti + 4, the activation operand with column gi's
// block; it reads back columns 2ti, 2ti+1 of rows gi, gi+8.  The part sums go
// to red[(p * rows_red + row) * kMT + token].
template <int NT, int F>
__device__ __forceinline__ void mma_task(const Gv& g, uint8_t* base, int r0, int p, int rows_red, int xrow, int n) {
  constexpr int BG = 8 / NT;  // blocks per group of 16 instructions
  const int lane = threadIdx.x & 31, gi = lane >> 2, ti = lane & 3;
  const int pb = p * g.pblk;  // first block of the part
  const int ngroups = (g.pblk + BG - 1) / BG;
  const uint8_t* rowa = base + g.codes + (size_t)(r0 + gi) * g.rstride + (size_t)pb * 16;
  const uint8_t* rowb = rowa + (size_t)8 * g.rstride;
  const uint32_t* sc = reinterpret_cast<const uint32_t*>(base + g.scales);
  const float* xinv = reinterpret_cast<const float*>(base + g.xinv);
  float acc[2][NT];
#pragma unroll
  for (int h = 0; h < 2; h++)
#pragma unroll
    for (int t = 0; t < NT; t++) acc[h][t] = 0.f;
  for (int gg = 0; gg < ngroups; gg++) {
    const int jb = gg * BG;
    const int ja = jb + ti / NT, jc = jb + (ti + 4) / NT;
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    const bool va = ja < g.pblk, vc = jc < g.pblk;
    const uint4 qa = va ? *reinterpret_cast<const uint4*>(rowa + ja * 16) : z;
    const uint4 qb = va ? *reinterpret_cast<const uint4*>(rowb + ja * 16) : z;
    const uint4 qc = vc ? *reinterpret_cast<const uint4*>(rowa + jc * 16) : z;
    const uint4 qd = vc ? *reinterpret_cast<const uint4*>(rowb + jc * 16) : z;
    uint32_t x0[16], x1[16];
    {
      const int j0 = jb + ti / NT, t0 = ti % NT, j1 = jb + (ti + 4) / NT, t1 = (ti + 4) % NT;
      load_xblock(g, base, gi == ti && j0 < g.pblk && t0 < n, xrow + t0, pb + j0, x0);
      load_xblock(g, base, gi == ti + 4 && j1 < g.pblk && t1 < n, xrow + t1, pb + j1, x1);
    }
    float d[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};
#define FT_MMA_STEP(I)                                                                                   \
  {                                                                                                      \
    const uint32_t a0 = code_pair<I>(qa), a1 = code_pair<I>(qb), a2 = code_pair<I>(qc),                 \
                   a3 = code_pair<I>(qd);                                                                \
    if (F == kFmtNv && I >= 8) mma16816(e, a0, a1, a2, a3, x0[I], x1[I]);                               \
    else mma16816(d, a0, a1, a2, a3, x0[I], x1[I]);                                                      \
  }
    FT_MMA_STEP(0) FT_MMA_STEP(1) FT_MMA_STEP(2) FT_MMA_STEP(3) FT_MMA_STEP(4) FT_MMA_STEP(5)
    FT_MMA_STEP(6) FT_MMA_STEP(7) FT_MMA_STEP(8) FT_MMA_STEP(9) FT_MMA_STEP(10) FT_MMA_STEP(11)
    FT_MMA_STEP(12) FT_MMA_STEP(13) FT_MMA_STEP(14) FT_MMA_STEP(15)
#undef FT_MMA_STEP
#pragma unroll
    for (int c = 0; c < 2; c++) {
      const int col = 2 * ti + c, j = jb + col / NT, tok = col % NT;
      if (j < g.pblk && tok < n) {
        const int blk = pb + j;
        const float xi = xinv[(xrow + tok) * g.chunks + blk];
#pragma unroll
        for (int h = 0; h < 2; h++) {
          const size_t row = (size_t)(r0 + gi + 8 * h);
          float v;
          if constexpr (F == kFmtNv) {
            const uint32_t sw = sc[row * g.sstride + (blk >> 1)] >> (16 * (blk & 1));
            v = fmaf(d[2 * h + c], e4m3_to_f32(sw & 0xffu), e[2 * h + c] * e4m3_to_f32((sw >> 8) & 0xffu)) * xi;
          } else {
            const uint32_t sw = sc[row * g.sstride + (blk >> 2)];
            v = d[2 * h + c] * (ue8m0_to_f32((sw >> (8 * (blk & 3))) & 0xffu) * xi);
          }
          acc[h][tok] += v;
        }
      }
    }
  }
  // the part sum of a row: its four lanes' sums, by xor shuffles
#pragma unroll
  for (int h = 0; h < 2; h++)
#pragma unroll
    for (int t = 0; t < NT; t++) {
      float a = acc[h][t];
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      acc[h][t] = a;
    }
  if (ti == 0) {
    float* red = reinterpret_cast<float*>(base + g.red);
#pragma unroll
    for (int h = 0; h < 2; h++)
#pragma unroll
      for (int t = 0; t < NT; t++)
        if (t < n) red[((size_t)p * rows_red + r0 + gi + 8 * h) * kMT + t] = acc[h][t];
  }
}

// Part sums of staged rows [0, rows) (a multiple of 16) into red (rows_red
// rows a part).  xr(q) gives the activations of 16-row group q: the first
// staged activation row and the token count (1 or 2).  Tasks (group, part)
// go to the warps in turn.
template <int F, class XR>
__device__ __forceinline__ void mma_dots(const Gv& g, uint8_t* base, int rows, int rows_red, XR xr) {
  const int warp = threadIdx.x >> 5;
  const int ntask = (rows >> 4) * g.parts;
  for (int task = warp; task < ntask; task += kWarps) {
    const int q = task / g.parts, p = task - q * g.parts;
    const int2 x = xr(q);
    if (x.y > 1) mma_task<2, F>(g, base, 16 * q, p, rows_red, x.x, x.y);
    else mma_task<1, F>(g, base, 16 * q, p, rows_red, x.x, x.y);
  }
}

// Partial sums of every row of the staged tile for n (<= kMT) tokens into red.
template <int F = kFmtMx>
__device__ __forceinline__ void tile_dots(const Gv& g, const LaneMap& m, uint8_t* base, int n) {
  if constexpr (F != kFmtBf16) {
    const int rows = g.nmat * g.R;
    mma_dots<F>(g, base, rows, rows, [n](int) { return make_int2(0, n); });
  } else {
    if (!m.on) return;
    float xf[kMT][32];
#pragma unroll
    for (int t = 0; t < kMT; t++) {
      if (m.c < g.chunks && t < n) load_act_bf16(g, base, t, m.c, xf[t]);
      else zero_act_bf16(xf[t]);
    }
    // rows per lane group and matrix, two at a time when that divides them
    // (32 fp32 activations per token leave room for two rows' chains; the
    // reduction tree does not depend on it)
    const int per = g.R % g.groups == 0 ? g.R / g.groups : 0;
    const int ru = (per % 2 == 0 && per > 0 && g.lpr >= 2) ? 2 : 1;
    if (n > 1) {
      if (ru == 2) tile_dots_t<2, 2>(g, m, base, xf);
      else tile_dots_t<1, 2>(g, m, base, xf);
    } else {
      if (ru == 2) tile_dots_t<2, 1>(g, m, base, xf);
      else tile_dots_t<1, 1>(g, m, base, xf);
    }
  }
}

// Row r of matrix mat for token t: the parts' partial sums in ascending order.
__device__ __forceinline__ float row_value(const Gv& g, const uint8_t* base, int mat, int r, int t) {
  const float* red = reinterpret_cast<const float*>(base + g.red);
  float s = red[((size_t)mat * g.R + r) * kMT + t];
  for (int p = 1; p < g.parts; p++) s += red[((size_t)(p * g.nmat + mat) * g.R + r) * kMT + t];
  return s;
}


constexpr uint64_t kSpinNs = 2000ull * 1000 * 1000;  // a dependency wait gives up after 2 s
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
  for (uint32_t n = 1;; n++) {
    if (mbar_try(bar, parity)) return true;
    // the global timer is read on every 32nd poll only
    if ((n & 31) == 0 && gclock() - t0 > kSpinNs) {
      set_status(status, kStTimeout);
      return false;
    }
  }
}
// One contiguous global -> shared copy by the bulk-copy engine, completing on bar.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void bulk_rows_warp(const Gv& g, uint8_t* dst, const uint8_t* src, int n, uint64_t* bar) {
  for (int r = threadIdx.x & 31; r < n; r += 32)
    bulk_g2s(dst + (size_t)r * g.rstride, src + (size_t)r * g.rowb, (uint32_t)g.rowb, bar);
}

// Thread 0 waits (acquire, bounded by limit_ns) until *p >= target, then the
// CTA synchronises; false (and the timeout status bit) when the wait gave up.
// `abort` is a shared flag, zero until a wait of this CTA gives up.
__device__ inline bool cta_wait_geq(const int* p, int target, int& abort, int* status, uint64_t limit_ns = kSpinNs) {
  if (threadIdx.x == 0 && ld_acquire(p) < target) {
    const uint64_t t0 = gclock();
    for (uint32_t n = 1; ld_acquire(p) < target; n++) {
      if ((n & 15) == 0 && gclock() - t0 > limit_ns) {
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


}  // namespace tile
}  // namespace ft

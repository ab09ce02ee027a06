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
// Other weight formats (fmt):
//   NVFP4  the same codes; a chunk has two E4M3 scales (16 elements each),
//          so its two halves keep separate sums, each times its scale; the
//          matrix's fp32 scale multiplies a row's value once, after the
//          reduction (by the caller).
//   BF16   a chunk is 32 bf16 weights (64 bytes); activations stay fp32 in
//          shared memory (no re-encoding: x and h enter exactly); each weight
//          widens to fp32 exactly and the products are summed by packed fp32
//          fused multiply-adds (fma.rn.f32x2) into two accumulators.
//
// Shared memory, from the tile's base:
//   codes  [nmat][R][rowb]       as in global memory (rowb = K/2, or 2K for BF16)
//   scales [nmat][R][atoms]      words of four scale bytes (K/128 words for
//                                MXFP4, K/64 for NVFP4, none for BF16)
//   xh     [kMT][4][K/32] x 16 B  activations, f16: quad i of chunk c at [t][i][c]
//          (BF16: [kMT][8][K/32] x 16 B of fp32)
//   xinv   [kMT][K/32]           inverse block factors (not for BF16)
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
  int fmt, rowb;      // weight format, bytes of a row's codes
  size_t codes, scales, xh, xinv, red, total;
};

__host__ __device__ inline Gv make_gv(int K, int rows, int nmat, int fmt = kFmtMx) {
  Gv g;
  g.K = K;
  g.nmat = nmat;
  g.fmt = fmt;
  g.rowb = fmt == kFmtBf16 ? 2 * K : K / 2;
  g.chunks = K / 32;
  g.atoms = fmt == kFmtMx ? K / 128 : fmt == kFmtNv ? K / 64 : 0;
  g.lpr = 1;
  while (g.lpr < 32 && g.lpr < g.chunks) g.lpr <<= 1;
  g.rpw = 32 / g.lpr;
  g.parts = (g.chunks + g.lpr - 1) / g.lpr;
  g.rsets = kWarps / g.parts;  // 0 for K > 16384: not supported
  g.groups = g.rsets * g.rpw;
  const int rmin = fmt == kFmtBf16 ? 2 : 8;
  int R = 128;
  while (R > rmin && (size_t)R * nmat * g.rowb > kTileBytes) R >>= 1;
  if (R > rows) R = rows;
  for (;;) {
    g.codes = 0;
    g.scales = (size_t)nmat * R * g.rowb;
    g.xh = g.scales + (size_t)nmat * R * g.atoms * 4;
    g.xinv = g.xh + (size_t)kMT * K * (fmt == kFmtBf16 ? 4 : 2);
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
  if (g.atoms == 0) return;  // BF16: no scales
  uint32_t* sd = reinterpret_cast<uint32_t*>(base + g.scales) + (size_t)mat * g.R * g.atoms;
  for (int i = threadIdx.x; i < g.R * g.atoms; i += kGemvThreads) {
    const int r = i / g.atoms, at = i - r * g.atoms;
    cp_async4(sd + i, sc_g + sf_word(row0 + r, at, g.atoms));
  }
}

// Stage rows [row0, row0 + R) of matrix `mat` (codes at codes_g, row pitch
// rowb; scale region sc_g) into the tile with cp.async.
__device__ __forceinline__ void stage_mat(const Gv& g, uint8_t* base, int mat, const uint8_t* codes_g,
                                          const uint8_t* sc_g, int row0) {
  uint8_t* dst = base + g.codes + (size_t)mat * g.R * g.rowb;
  const uint8_t* src = codes_g + (size_t)row0 * g.rowb;
  const int n16 = g.R * (g.rowb / 16);
  for (int i = threadIdx.x; i < n16; i += kGemvThreads) cp_async16(dst + (size_t)i * 16, src + (size_t)i * 16);
  stage_scales(g, base, mat, sc_g, row0);
}

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
  q = *reinterpret_cast<const uint4*>(codes + (size_t)row * g.rowb + c * 16);
  const uint32_t sw = sc[(size_t)row * g.atoms + (c >> 2)];
  s = ue8m0_to_f32((sw >> (8 * (c & 3))) & 0xffu);
}

// NVFP4: the codes of chunk c and the E4M3 scales of its two 16-element
// halves (adjacent bytes of one scale word: blocks 2c and 2c + 1).
__device__ __forceinline__ void tile_chunk_nv(const Gv& g, const uint8_t* codes, const uint32_t* sc, int row, int c,
                                              uint4& q, float& s0, float& s1) {
  q = *reinterpret_cast<const uint4*>(codes + (size_t)row * g.rowb + c * 16);
  const uint32_t sw = sc[(size_t)row * g.atoms + (c >> 1)] >> (16 * (c & 1));
  s0 = e4m3_to_f32(sw & 0xffu);
  s1 = e4m3_to_f32((sw >> 8) & 0xffu);
}

// BF16: the 32 weights (64 bytes) of chunk c of staged row `row`.
__device__ __forceinline__ void tile_chunk_bf16(const Gv& g, const uint8_t* codes, int row, int c, uint4 (&q)[4]) {
  const uint4* p = reinterpret_cast<const uint4*>(codes + (size_t)row * g.rowb + c * 64);
#pragma unroll
  for (int i = 0; i < 4; i++) q[i] = p[i];
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

// NVFP4: the dot of a chunk's two 16-element halves, kept apart (words 0-1
// and 2-3 of the codes), each a chain of fused multiply-adds in fixed order.
template <int NT>
__device__ __forceinline__ void chunk_dot_nv(uint4 q, const uint32_t (&x)[kMT][16], float* d0, float* d1) {
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
      for (int t = 0; t < NT; t++) acc[t][wv >> 1] = fma_f16x2(h[j], x[t][4 * wv + j], acc[t][wv >> 1]);
  }
#pragma unroll
  for (int t = 0; t < NT; t++) {
    d0[t] = acc[t][0];
    d1[t] = acc[t][1];
  }
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

// The same reduction over eight rows v[0..7]: a first exchange step keeps
// four of them, then the four-row steps.  Lanes pair by the same bits in the
// same order as above, so every row's sum is bit for bit the one a smaller
// step gives.  Needs lpr >= 8; returns the row this lane holds.
template <int NT>
__device__ __forceinline__ int group_reduce8(float (&v)[8][kMT], int lpr) {
  const int lane = threadIdx.x & 31;
  int d = lpr >> 1;
  const bool hi = lane & d;
#pragma unroll
  for (int t = 0; t < NT; t++)
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const float sd = hi ? v[i][t] : v[4 + i][t], kp = hi ? v[4 + i][t] : v[i][t];
      v[i][t] = kp + __shfl_xor_sync(0xffffffffu, sd, d);
    }
  int row = hi ? 4 : 0;
  d >>= 1;
  {
    const bool h2 = lane & d;
#pragma unroll
    for (int t = 0; t < NT; t++) {
      const float s0 = h2 ? v[0][t] : v[2][t], s1 = h2 ? v[1][t] : v[3][t];
      const float k0 = h2 ? v[2][t] : v[0][t], k1 = h2 ? v[3][t] : v[1][t];
      v[0][t] = k0 + __shfl_xor_sync(0xffffffffu, s0, d);
      v[1][t] = k1 + __shfl_xor_sync(0xffffffffu, s1, d);
    }
    row += h2 ? 2 : 0;
    d >>= 1;
  }
  {
    const bool h3 = lane & d;
#pragma unroll
    for (int t = 0; t < NT; t++) {
      const float sd = h3 ? v[0][t] : v[1][t], kp = h3 ? v[1][t] : v[0][t];
      v[0][t] = kp + __shfl_xor_sync(0xffffffffu, sd, d);
    }
    row += h3 ? 1 : 0;
    d >>= 1;
  }
  for (; d >= 1; d >>= 1)
#pragma unroll
    for (int t = 0; t < NT; t++) v[0][t] += __shfl_xor_sync(0xffffffffu, v[0][t], d);
  return row;
}

// Value of chunk c of staged row `row` for NT tokens, before the row's
// reduction over its lanes: MXFP4 chunk sum x (scale x inverse factor);
// NVFP4 (half sum x scale, added) x inverse factor; BF16 the fp32 dot.
template <int NT, int F>
__device__ __forceinline__ void chunk_value(const Gv& g, const uint8_t* codes, const uint32_t* sc, int row, int c,
                                            const uint32_t (&x)[kMT][16], const float (&xi)[kMT],
                                            const float (&xf)[kMT][32], float* v) {
  if constexpr (F == kFmtMx) {
    uint4 q;
    float s;
    tile_chunk(g, codes, sc, row, c, q, s);
    float d[NT];
    chunk_dot<NT>(q, x, d);
#pragma unroll
    for (int t = 0; t < NT; t++) v[t] = d[t] * (s * xi[t]);
  } else if constexpr (F == kFmtNv) {
    uint4 q;
    float s0, s1;
    tile_chunk_nv(g, codes, sc, row, c, q, s0, s1);
    float d0[NT], d1[NT];
    chunk_dot_nv<NT>(q, x, d0, d1);
#pragma unroll
    for (int t = 0; t < NT; t++) v[t] = fmaf(d0[t], s0, d1[t] * s1) * xi[t];
  } else {
    uint4 q[4];
    tile_chunk_bf16(g, codes, row, c, q);
    chunk_dot_bf16<NT>(q, xf, v);
  }
}

// Activations of staged row srow, chunk c, into one token slot of the lane's
// registers (f16 pairs and the inverse factor; fp32 for BF16 weights).
template <int F>
__device__ __forceinline__ void load_act(const Gv& g, const uint8_t* base, int srow, int c, uint32_t (&x)[16],
                                         float& xi, float (&xf)[32]) {
  if constexpr (F == kFmtBf16) {
    const float4* p = reinterpret_cast<const float4*>(base + g.xh);
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const float4 f = p[((size_t)srow * 8 + i) * g.chunks + c];
      xf[4 * i] = f.x;
      xf[4 * i + 1] = f.y;
      xf[4 * i + 2] = f.z;
      xf[4 * i + 3] = f.w;
    }
  } else {
    const uint4* xh = reinterpret_cast<const uint4*>(base + g.xh);
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const uint4 u = xh[(size_t)srow * (g.K / 8) + (size_t)i * g.chunks + c];
      x[4 * i] = u.x;
      x[4 * i + 1] = u.y;
      x[4 * i + 2] = u.z;
      x[4 * i + 3] = u.w;
    }
    xi = reinterpret_cast<const float*>(base + g.xinv)[srow * g.chunks + c];
  }
}

template <int F>
__device__ __forceinline__ void zero_act(uint32_t (&x)[16], float& xi, float (&xf)[32]) {
  if constexpr (F == kFmtBf16) {
#pragma unroll
    for (int i = 0; i < 32; i++) xf[i] = 0.f;
  } else {
#pragma unroll
    for (int i = 0; i < 16; i++) x[i] = 0u;
    xi = 0.f;
  }
}

// Partial sums of the staged tile's rows for NT tokens into red.  Lane group
// grp takes rows grp + j*groups, RU of them at a time.
template <int RU, int NT, int F>
__device__ __forceinline__ void tile_dots_t(const Gv& g, const LaneMap& m, uint8_t* base,
                                            const uint32_t (&x)[kMT][16], const float (&xi)[kMT],
                                            const float (&xf)[kMT][32]) {
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
        if (cv) chunk_value<NT, F>(g, codes, sc, mat * g.R + m.grp + (j0 + u) * g.groups, m.c, x, xi, xf, v[u]);
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

// A two-matrix tile with R = 4 * groups in one step of eight rows per lane
// group (rows grp + j*groups of both matrices, j < 4).
template <int NT, int F>
__device__ __forceinline__ void tile_dots_fused8(const Gv& g, const LaneMap& m, uint8_t* base,
                                                 const uint32_t (&x)[kMT][16], const float (&xi)[kMT],
                                                 const float (&xf)[kMT][32]) {
  const uint8_t* codes = base + g.codes;
  const uint32_t* sc = reinterpret_cast<const uint32_t*>(base + g.scales);
  float* red = reinterpret_cast<float*>(base + g.red);
  const bool cv = m.c < g.chunks;
  float v[8][kMT];
#pragma unroll
  for (int u = 0; u < 8; u++) {
    v[u][0] = v[u][1] = 0.f;
    if (cv) chunk_value<NT, F>(g, codes, sc, (u >> 2) * g.R + m.grp + (u & 3) * g.groups, m.c, x, xi, xf, v[u]);
  }
  const int u = group_reduce8<NT>(v, g.lpr);
  if (((threadIdx.x & 31) & ((g.lpr >> 3) - 1)) == 0) {
    const int mat = u >> 2, r = m.grp + (u & 3) * g.groups;
    float* o = red + ((size_t)(m.part * g.nmat + mat) * g.R + r) * kMT;
#pragma unroll
    for (int t = 0; t < NT; t++) o[t] = v[0][t];
  }
}

// Partial sums of every row of the staged tile for n (<= kMT) tokens into red.
// NTF, RUF: tokens per pass and rows per step fixed at compile time (a build
// for one tile shape and batch carries only that loop), or 0 for the choice
// at run time; a fixed NTF = 1 takes n = 1 only; RUF = 8 takes a two-matrix
// tile with R = 4 * groups in one step.
template <int F = kFmtMx, int NTF = 0, int RUF = 0>
__device__ __forceinline__ void tile_dots(const Gv& g, const LaneMap& m, uint8_t* base, int n) {
  if (!m.on) return;
  uint32_t x[kMT][16];
  float xi[kMT] = {0.f, 0.f};
  float xf[kMT][32];
#pragma unroll
  for (int t = 0; t < kMT; t++) {
    if (m.c < g.chunks && t < n) load_act<F>(g, base, t, m.c, x[t], xi[t], xf[t]);
    else zero_act<F>(x[t], xi[t], xf[t]);
  }
  // rows per lane group and matrix; groups of 4 or 2 when they divide it
  // (BF16 holds 32 fp32 activations per token: at most 2 rows at a time, so
  // that the registers suffice; the reduction tree does not depend on it)
  const int per = g.R % g.groups == 0 ? g.R / g.groups : 0;
  const int ru = RUF ? RUF
                 : (F != kFmtBf16 && per % 4 == 0 && per > 0 && g.lpr >= 4) ? 4
                 : (per % 2 == 0 && per > 0 && g.lpr >= 2)                ? 2
                                                                           : 1;
  if constexpr (NTF == 1 && RUF == 8) {  // both matrices of a gate/up tile in one step
    tile_dots_fused8<1, F>(g, m, base, x, xi, xf);
    return;
  } else if constexpr (NTF == 1 && RUF != 0) {
    tile_dots_t<RUF, 1, F>(g, m, base, x, xi, xf);
    return;
  }
  if (NTF != 1 && n > 1) {
    if (ru == 4) tile_dots_t<4, 2, F>(g, m, base, x, xi, xf);
    else if (ru == 2) tile_dots_t<2, 2, F>(g, m, base, x, xi, xf);
    else tile_dots_t<1, 2, F>(g, m, base, x, xi, xf);
  } else {
    if (ru == 4) tile_dots_t<4, 1, F>(g, m, base, x, xi, xf);
    else if (ru == 2) tile_dots_t<2, 1, F>(g, m, base, x, xi, xf);
    else tile_dots_t<1, 1, F>(g, m, base, x, xi, xf);
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

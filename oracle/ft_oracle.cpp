// ft_oracle.cpp — CPU oracle of one FreeToken-style MoE layer forward pass
// with an expert cache, in plain C++17 and fp64.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
// CPU-baseline / reference legs of bench.py may load liboracle.so.  It shares
// no code with the CUDA library and includes none of its headers; the two
// meet only through the seeded inputs of synth/.  It restates, in plain loops,
// the same definitions as the numpy oracle beside it (oracle/*.py), which
// serves as its cross-check.
//
// Sources (page, section):
//   - a gate picks a few experts per token and layer (aiforradalom.hu, "A
//     Mixture-of-Experts (MoE) kihívásai és a FreeToken megoldásai": 6 of 256
//     per layer for DeepSeek-V4-Flash);
//   - experts run on the GPU from weights held there or fetched over PCIe and
//     their partial results are summed with no approximation; one global LRU
//     cache spans the MoE layers (jansverre.net, "Hvorfor er båndbredden
//     viktigere enn antall kjerner?");
//   - MXFP4 weights (jansverre.net, "Hvor raskt kjører modellene?"): e2m1
//     elements with one power-of-two (UE8M0) scale per 32 (the OCP MX
//     format); BF16 and NVFP4 builds of Qwen3.6-35B-A3B (same section);
//   - the shared LRU exploits adjacent tokens' expert overlap, and the GPU
//     cache can be resized without reloading the host pool (aipolix.com,
//     paragraphs on semantic-aware caching and on elastic memory management).
// Readings where the pages are silent (softmax top-k with ties to the lower
// id, SwiGLU experts, the fixed router summation order, the quantiser, the
// LRU tie rules) are the ones the numpy oracle states, restated here.
//
// Build: g++ -O2 -std=c++17 -fPIC -shared -fopenmp (oracle/build.py).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <list>
#include <map>
#include <utility>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

#define FTO_API extern "C" __attribute__((visibility("default")))

namespace {

// ---------------------------------------------------------------------------
// element and scale decoding (OCP MX: e2m1 = sign, 2 exponent bits with bias
// 1, 1 mantissa bit; exponent 0 encodes 0.5 * m; UE8M0 byte e = 2^(e - 127),
// 255 = NaN)
// ---------------------------------------------------------------------------
double e2m1(int code) {
  const int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  const double mag = e == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;  // code 8 gives -0.0
}

double ue8m0(int byte) { return byte == 255 ? NAN : std::ldexp(1.0, byte - 127); }

// E4M3 without infinities: sign, 4 exponent bits (bias 7), 3 fraction bits;
// exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN.
double e4m3(int byte) {
  const int s = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
  if (e == 15 && m == 7) return NAN;
  const double mag = e == 0 ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

int64_t pad(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// Byte offset, inside a matrix's scale region, of the scale of block `kb` of
// `row` (blocks of 32 elements for MXFP4, 16 for NVFP4): atoms of 128 rows x 4
// blocks in 512 bytes, row r in the 16-byte group r % 32, the 4-byte word
// (r % 128) / 32, the byte kb % 4; atoms along K first.
int64_t scale_index(int64_t row, int64_t kb, int64_t n_kblocks) {
  const int64_t atoms_k = pad(n_kblocks, 4) / 4;
  const int64_t atom = (row / 128) * atoms_k + kb / 4;
  return atom * 512 + (row % 32) * 16 + ((row % 128) / 32) * 4 + kb % 4;
}

struct Layout {
  int64_t wg, wu, wd, wg_sf, wu_sf, wd_sf, used, stride, tensor_scales;
};

// MXFP4 blob: codes Wg [I][H/2], Wu [I][H/2], Wd [H][I/2] (element 2i in the
// low nibble), then the three scale regions in whole atoms, zero padded to a
// multiple of 256 bytes.
Layout mx_layout(int H, int I) {
  Layout L{};
  L.wg = 0;
  L.wu = (int64_t)I * H / 2;
  L.wd = 2 * L.wu;
  const int64_t end = L.wd + (int64_t)H * I / 2;
  const int64_t gu = pad(I, 128) * pad(H / 32, 4), d = pad(H, 128) * pad(I / 32, 4);
  L.wg_sf = end;
  L.wu_sf = end + gu;
  L.wd_sf = end + 2 * gu;
  L.used = end + 2 * gu + d;
  L.stride = pad(L.used, 256);
  return L;
}

// NVFP4 blob: the MXFP4 code regions, E4M3 scale regions of 16-element
// blocks in the same atoms, three fp32 matrix scales and 4 zero bytes.
Layout nv_layout(int H, int I) {
  Layout L{};
  L.wg = 0;
  L.wu = (int64_t)I * H / 2;
  L.wd = (int64_t)I * H;
  const int64_t end = (int64_t)I * H + (int64_t)H * I / 2;
  const int64_t gu = pad(I, 128) * pad(H / 16, 4), d = pad(H, 128) * pad(I / 16, 4);
  L.wg_sf = end;
  L.wu_sf = end + gu;
  L.wd_sf = end + 2 * gu;
  L.tensor_scales = end + 2 * gu + d;
  L.used = L.tensor_scales + 16;
  L.stride = pad(L.used, 256);
  return L;
}

enum Format { kMx = 0, kNv = 1, kBf16 = 2 };

// Matrix mat (0 Wg [I][H], 1 Wu [I][H], 2 Wd [H][I]) of a blob as fp64.
std::vector<double> weight_matrix(const uint8_t* blob, int H, int I, int mat, int fmt) {
  const int rows = mat < 2 ? I : H, K = mat < 2 ? H : I;
  std::vector<double> w((size_t)rows * K);
  if (fmt == kBf16) {
    const int64_t off = (int64_t)mat * 2 * I * H;  // Wg, Wu, Wd, each rows x K bf16
    for (int64_t i = 0; i < (int64_t)rows * K; i++)
      w[i] = bf16_to_double((uint16_t)(blob[off + 2 * i] | (blob[off + 2 * i + 1] << 8)));
    return w;
  }
  const Layout L = fmt == kMx ? mx_layout(H, I) : nv_layout(H, I);
  const int64_t co = mat == 0 ? L.wg : mat == 1 ? L.wu : L.wd;
  const int64_t so = mat == 0 ? L.wg_sf : mat == 1 ? L.wu_sf : L.wd_sf;
  const int blk = fmt == kMx ? 32 : 16;
  double ts = 1.0;
  if (fmt == kNv) {
    float f;
    std::memcpy(&f, blob + L.tensor_scales + 4 * mat, 4);
    ts = (double)f;
  }
  for (int r = 0; r < rows; r++)
    for (int kk = 0; kk < K; kk++) {
      const uint8_t byte = blob[co + (int64_t)r * (K / 2) + kk / 2];
      const int code = (kk & 1) ? (byte >> 4) : (byte & 15);
      const uint8_t sb = blob[so + scale_index(r, kk / blk, K / blk)];
      const double scale = fmt == kMx ? ue8m0(sb) : e4m3(sb) * ts;
      w[(size_t)r * K + kk] = e2m1(code) * scale;
    }
  return w;
}

// ---------------------------------------------------------------------------
// OCP MX quantiser of one block of 32 values: scale byte = floor(log2 amax)
// - 2 (the largest e2m1 exponent) + 127, clamped to [0, 254] (amax = 0 gives
// 0); each value / scale rounded to the nearest e2m1 magnitude, ties to the
// even code, saturating at 6; the sign kept (a negative value that rounds to
// zero is code 8).
// ---------------------------------------------------------------------------
const double kGrid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

int round_to_grid(double a) {
  if (a >= 6.0) return 7;
  int best = 0;
  double bd = std::fabs(a - kGrid[0]);
  for (int c = 1; c < 8; c++) {
    const double d = std::fabs(a - kGrid[c]);
    if (d < bd || (d == bd && (c & 1) == 0 && (best & 1) != 0)) {
      bd = d;
      best = c;
    }
  }
  return best;
}

int block_scale_byte(double amax) {
  if (amax == 0.0) return 0;
  int ex;
  std::frexp(amax, &ex);  // amax = m * 2^ex, m in [0.5, 1)
  return std::min(std::max((ex - 1) + 127 - 2, 0), 254);
}

// Quantise and dequantise one row of K values in place (fp64 in, fp64 out).
void mx_roundtrip(double* v, int K) {
  for (int b = 0; b < K; b += 32) {
    double amax = 0.0;
    for (int i = 0; i < 32; i++) amax = std::max(amax, std::fabs(v[b + i]));
    const int e = block_scale_byte(amax);
    const double inv = std::ldexp(1.0, 127 - e), sc = std::ldexp(1.0, e - 127);
    for (int i = 0; i < 32; i++) {
      const double x = v[b + i];
      const int code = round_to_grid(std::fabs(x) * inv) | (std::signbit(x) ? 8 : 0);
      v[b + i] = e2m1(code) * sc;
    }
  }
}

// ---------------------------------------------------------------------------
// NVFP4 activations (the prefill path of NVFP4 experts).  The pages leave
// activation scaling open; the reading is the two-level one: a per-tensor
// scale s = amax / 2688 over the matrix a GEMM reads (all tokens of x; every
// h row of the layer), E4M3 block scales per 16 values, e2m1 codes.  Each
// step decides a byte, so each is one fp32 operation rounded to nearest even:
//   s = amax / 2688 (0 when amax < 2^-100: every byte 0), g = 1 / (s * 6);
//   per block e = E4M3(amax_block * g) (nearest, ties to the even byte, at
//   most 448), dq = value(e) * s, r = 1 / dq, code = e2m1(v * r) (dq == 0:
//   codes 0).  Dequantised value: code x value(e) x s.
// ---------------------------------------------------------------------------
int e4m3_round(float v) {
  if (v >= 448.0f) return 0x7E;
  int best = 0;
  double bd = std::fabs((double)v - e4m3(0));
  for (int b = 1; b < 0x7F; b++) {
    const double d = std::fabs((double)v - e4m3(b));
    if (d < bd || (d == bd && (b & 1) == 0 && (best & 1) != 0)) {
      bd = d;
      best = b;
    }
  }
  return best;
}

struct NvScale {
  float s, g;
};

NvScale nv_tensor_scale(float amax) {
  NvScale t{0.0f, 0.0f};
  if (amax >= 0x1p-100f) {
    t.s = amax / 2688.0f;
    t.g = 1.0f / (t.s * 6.0f);
  }
  return t;
}

// One row of K values (exact in fp32): codes [K] and scale bytes [K/16] (each
// optional) and the dequantised row in fp64.
void nv_quantize_row(const float* v, int K, NvScale t, uint8_t* codes, uint8_t* scales, double* deq) {
  for (int b = 0; b < K; b += 16) {
    int e = 0;
    if (t.s != 0.0f) {
      float amax = 0.0f;
      for (int i = 0; i < 16; i++) amax = std::max(amax, std::fabs(v[b + i]));
      e = e4m3_round(amax * t.g);
    }
    const float dq = (float)e4m3(e) * t.s;
    const float r = dq > 0.0f ? 1.0f / dq : 0.0f;
    for (int i = 0; i < 16; i++) {
      int code = 0;
      if (dq > 0.0f) {
        const float q = v[b + i] * r;
        code = round_to_grid(std::fabs((double)q)) | (std::signbit(q) ? 8 : 0);
      }
      if (codes) codes[b + i] = (uint8_t)code;
      if (deq) deq[b + i] = e2m1(code) * e4m3(e) * (double)t.s;
    }
    if (scales) scales[b / 16] = (uint8_t)e;
  }
}

// fp64 -> bf16 bits, nearest with ties to even, directly (no fp32 step).
uint16_t round_bf16(double x) {
  if (std::isnan(x)) return 0x7FC0;
  const uint16_t sign = std::signbit(x) ? 0x8000 : 0;
  const double a = std::fabs(x);
  if (a == 0.0) return sign;
  int ex;
  std::frexp(a, &ex);                          // a in [2^(ex-1), 2^ex)
  const int q_exp = std::max(ex - 1, -126) - 7;  // bf16 ulp; subnormals at 2^-133
  const double q = std::ldexp(a, -q_exp);      // exact
  double r = std::floor(q);
  const double frac = q - r;
  if (frac > 0.5 || (frac == 0.5 && std::fmod(r, 2.0) == 1.0)) r += 1.0;
  const double val = std::ldexp(r, q_exp);
  if (val >= std::ldexp(1.0, 128)) return sign | 0x7F80;
  const float f = (float)val;  // exact: val has at most 8 significant bits
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return sign | (uint16_t)(u >> 16);
}

double silu(double z) { return z / (1.0 + std::exp(-z)); }

// ---------------------------------------------------------------------------
// routing
// ---------------------------------------------------------------------------

// logit[t][e] = x[t] . Wr[e] in a fixed order: element kk joins partial sum
// (kk / 4) % 32, each partial sum in ascending kk; the 32 partial sums meet
// in a butterfly with distances 16, 8, 4, 2, 1 (position p adds position
// p xor d); position 0 is rounded once to fp32.  Each bf16 x fp32 product is
// exact in fp64.
void router_logits(const uint16_t* x, const float* wr, int T, int H, int E, float* out) {
  for (int t = 0; t < T; t++)
    for (int e = 0; e < E; e++) {
      double part[32] = {0};
      for (int kk = 0; kk < H; kk++)
        part[(kk / 4) % 32] += bf16_to_double(x[(size_t)t * H + kk]) * (double)wr[(size_t)e * H + kk];
      for (int d = 16; d >= 1; d >>= 1) {
        double nxt[32];
        for (int p = 0; p < 32; p++) nxt[p] = part[p] + part[p ^ d];
        std::memcpy(part, nxt, sizeof part);
      }
      out[(size_t)t * E + e] = (float)part[0];
    }
}

// Rank of a logit: larger ranks first; NaN ranks below -inf; -0 equals +0.
bool ranks_before(float a, int ia, float b, int ib) {
  const bool na = std::isnan(a), nb = std::isnan(b);
  if (na != nb) return nb;        // a number before a NaN
  if (!na && a != b) return a > b;
  return ia < ib;                 // equal values (or both NaN): lower id first
}

// ids [T][k] in rank order; returns 1 if a logit is NaN or +inf or a row has
// no finite logit.
int topk(const float* lg, int T, int E, int k, int32_t* ids) {
  int bad = 0;
  std::vector<int> order(E);
  for (int t = 0; t < T; t++) {
    const float* row = lg + (size_t)t * E;
    bool any_finite = false;
    for (int e = 0; e < E; e++) {
      if (std::isnan(row[e]) || row[e] == INFINITY) bad = 1;
      if (std::isfinite(row[e])) any_finite = true;
    }
    if (!any_finite) bad = 1;
    for (int e = 0; e < E; e++) order[e] = e;
    std::sort(order.begin(), order.end(), [&](int a, int b) { return ranks_before(row[a], a, row[b], b); });
    for (int j = 0; j < k; j++) ids[(size_t)t * k + j] = order[j];
  }
  return bad;
}

// w[t][j] = p[ids[t][j]] with p the softmax of the row over all E (fp64),
// divided by the sum over the k chosen when renorm.
void softmax_weights(const float* lg, const int32_t* ids, int T, int E, int k, int renorm, double* w) {
  std::vector<double> p(E);
  for (int t = 0; t < T; t++) {
    const float* row = lg + (size_t)t * E;
    double m = -INFINITY;
    for (int e = 0; e < E; e++) m = std::max(m, (double)row[e]);
    double z = 0.0;
    for (int e = 0; e < E; e++) {
      p[e] = std::exp((double)row[e] - m);
      z += p[e];
    }
    double sel = 0.0;
    for (int j = 0; j < k; j++) sel += p[ids[(size_t)t * k + j]] / z;
    for (int j = 0; j < k; j++) {
      const double pj = p[ids[(size_t)t * k + j]] / z;
      w[(size_t)t * k + j] = renorm ? pj / sel : pj;
    }
  }
}

// Stable sort of the pairs f = t*k + j by expert id.
void permutation(const int32_t* ids, int P, int E, int32_t* offs, int32_t* perm, int32_t* inv) {
  std::vector<int> f(P);
  for (int i = 0; i < P; i++) f[i] = i;
  std::stable_sort(f.begin(), f.end(), [&](int a, int b) { return ids[a] < ids[b]; });
  for (int pos = 0; pos < P; pos++) {
    perm[pos] = f[pos];
    inv[f[pos]] = pos;
  }
  for (int e = 0; e <= E; e++) offs[e] = 0;
  for (int i = 0; i < P; i++) offs[ids[i] + 1]++;
  for (int e = 0; e < E; e++) offs[e + 1] += offs[e];
}

// ---------------------------------------------------------------------------
// expert FFN: y = Wd (silu(Wg x) * (Wu x)), fp64; in MXFP4-activation mode x
// and h are quantised per 32 (OCP MX) before their products
// ---------------------------------------------------------------------------
void expert_ffn(const uint8_t* blob, int H, int I, const double* x, int m, int mxfp4, int fmt, double* y) {
  const std::vector<double> wg = weight_matrix(blob, H, I, 0, fmt);
  const std::vector<double> wu = weight_matrix(blob, H, I, 1, fmt);
  const std::vector<double> wd = weight_matrix(blob, H, I, 2, fmt);
  std::vector<double> xs(H), h(I);
  for (int t = 0; t < m; t++) {
    std::copy(x + (size_t)t * H, x + (size_t)(t + 1) * H, xs.begin());
    if (mxfp4) mx_roundtrip(xs.data(), H);
    for (int i = 0; i < I; i++) {
      double g = 0.0, u = 0.0;
      for (int kk = 0; kk < H; kk++) {
        g += wg[(size_t)i * H + kk] * xs[kk];
        u += wu[(size_t)i * H + kk] * xs[kk];
      }
      h[i] = silu(g) * u;
    }
    if (mxfp4) mx_roundtrip(h.data(), I);
    for (int n = 0; n < H; n++) {
      double acc = 0.0;
      for (int i = 0; i < I; i++) acc += wd[(size_t)n * I + i] * h[i];
      y[(size_t)t * H + n] = acc;
    }
  }
}

// ---------------------------------------------------------------------------
// global LRU over (layer, expert) keys
// ---------------------------------------------------------------------------
struct Lru {
  int64_t capacity;
  std::list<std::pair<int, int>> order;          // least recent first
  std::map<std::pair<int, int>, int> slot;
  // decode-time next-layer prefetch (off while per_layer == 0)
  int n_layers = 0, n_experts = 0, per_layer = 0;
  std::vector<int64_t> count;                    // [layer][expert] steps whose set held the expert
  std::map<std::pair<int, int>, int> unused;     // prefetched keys not hit yet
  int64_t prefetches = 0, prefetch_hits = 0;
};

}  // namespace

// ===========================================================================
// C ABI (ctypes)
// ===========================================================================

FTO_API int fto_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

FTO_API void fto_e2m1_table(double* out16) {
  for (int c = 0; c < 16; c++) out16[c] = e2m1(c);
}

FTO_API void fto_ue8m0_table(double* out256) {
  for (int b = 0; b < 256; b++) out256[b] = ue8m0(b);
}

FTO_API void fto_e4m3_table(double* out256) {
  for (int b = 0; b < 256; b++) out256[b] = e4m3(b);
}

FTO_API int64_t fto_scale_index(int64_t row, int64_t kb, int64_t n_kblocks) { return scale_index(row, kb, n_kblocks); }

// out[0..7] = wg, wu, wd, wg_sf, wu_sf, wd_sf, used, stride of the MXFP4
// blob (fmt 0) or the NVFP4 blob (fmt 1; out[8] = tensor_scales)
FTO_API void fto_layout(int H, int I, int fmt, int64_t* out) {
  const Layout L = fmt == kMx ? mx_layout(H, I) : nv_layout(H, I);
  const int64_t v[9] = {L.wg, L.wu, L.wd, L.wg_sf, L.wu_sf, L.wd_sf, L.used, L.stride, L.tensor_scales};
  std::memcpy(out, v, sizeof v);
}

FTO_API void fto_weight_matrix(const uint8_t* blob, int H, int I, int mat, int fmt, double* out) {
  const std::vector<double> w = weight_matrix(blob, H, I, mat, fmt);
  std::copy(w.begin(), w.end(), out);
}

// codes [R][K] (one code per element) and scale bytes [R][K/32]
FTO_API void fto_quantize_rows(const double* x, int64_t R, int K, uint8_t* codes, uint8_t* scales) {
  for (int64_t r = 0; r < R; r++)
    for (int b = 0; b < K; b += 32) {
      const double* v = x + r * K + b;
      double amax = 0.0;
      for (int i = 0; i < 32; i++) amax = std::max(amax, std::fabs(v[i]));
      const int e = block_scale_byte(amax);
      scales[r * (K / 32) + b / 32] = (uint8_t)e;
      const double inv = std::ldexp(1.0, 127 - e);
      for (int i = 0; i < 32; i++)
        codes[r * K + b + i] = (uint8_t)(round_to_grid(std::fabs(v[i]) * inv) | (std::signbit(v[i]) ? 8 : 0));
    }
}

// NVFP4 rows: x [R][K] (values exact in fp32) -> codes [R][K] (one code per
// element), scale bytes [R][K/16]; returns the per-tensor scale (from the
// largest |x| when s_in < 0, else s_in).
FTO_API float fto_nvfp4_quantize_rows(const double* x, int64_t R, int K, float s_in, uint8_t* codes, uint8_t* scales) {
  std::vector<float> v((size_t)R * K);
  float amax = 0.0f;
  for (size_t i = 0; i < v.size(); i++) {
    v[i] = (float)x[i];
    amax = std::max(amax, std::fabs(v[i]));
  }
  NvScale t = nv_tensor_scale(amax);
  if (s_in >= 0.0f) t = s_in > 0.0f ? NvScale{s_in, 1.0f / (s_in * 6.0f)} : NvScale{0.0f, 0.0f};
  for (int64_t r = 0; r < R; r++) nv_quantize_row(v.data() + r * K, K, t, codes + r * K, scales + r * (K / 16), nullptr);
  return t.s;
}

FTO_API void fto_round_bf16(const double* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = round_bf16(v[i]);
}

FTO_API void fto_router_logits(const uint16_t* x, const float* wr, int T, int H, int E, float* out) {
  router_logits(x, wr, T, H, E, out);
}

FTO_API int fto_topk(const float* lg, int T, int E, int k, int32_t* ids) { return topk(lg, T, E, k, ids); }

FTO_API void fto_softmax_weights(const float* lg, const int32_t* ids, int T, int E, int k, int renorm, double* w) {
  softmax_weights(lg, ids, T, E, k, renorm, w);
}

FTO_API void fto_permutation(const int32_t* ids, int P, int E, int32_t* offs, int32_t* perm, int32_t* inv) {
  permutation(ids, P, E, offs, perm, inv);
}

FTO_API void fto_expert_ffn(const uint8_t* blob, int H, int I, const double* x, int m, int mxfp4, int fmt, double* y) {
  expert_ffn(blob, H, I, x, m, mxfp4, fmt, y);
}

// One MoE layer on T tokens:
//   out[t] = sum_j w[t][j] FFN_{ids[t][j]}(x[t]) (+ shared FFN(x[t])), summed
//   over j ascending, then the shared expert, in fp64; out_bits = bf16.
//   blobs [E] pointers (only the selected experts are read), shared NULL or
//   a blob; logits [T][E] or NULL (then router_w [E][H] and router_logits).
//   Experts run in parallel on `threads` OpenMP threads (1 = serial; the sum
//   order of the combine does not depend on it).  ids / w outputs may be NULL.
//   mxfp4 selects the activations: 0 as given (decode), 1 MXFP4 per row, 2
//   NVFP4 with the per-tensor scales of x (all T tokens) and of h (every h
//   row of the layer, so all units' h come before any down projection).
// Returns 1 if the routing saw a NaN / +inf logit (as topk), else 0.
FTO_API int fto_moe_layer(const uint16_t* x_bits, int T, int H, int I, int E, int k, const uint8_t* const* blobs,
                          const uint8_t* shared, const float* logits, const float* router_w, int renorm, int mxfp4,
                          int fmt, int threads, double* out, uint16_t* out_bits, int32_t* ids_out, double* w_out) {
  std::vector<float> lg((size_t)T * E);
  if (logits) std::copy(logits, logits + (size_t)T * E, lg.begin());
  else router_logits(x_bits, router_w, T, H, E, lg.data());
  std::vector<int32_t> ids((size_t)T * k);
  const int bad = topk(lg.data(), T, E, k, ids.data());
  std::vector<double> w((size_t)T * k);
  softmax_weights(lg.data(), ids.data(), T, E, k, renorm, w.data());
  std::vector<double> x((size_t)T * H);
  for (size_t i = 0; i < x.size(); i++) x[i] = bf16_to_double(x_bits[i]);
  // units: the distinct selected experts (ascending), then the shared expert
  std::vector<int> units(ids.begin(), ids.end());
  std::sort(units.begin(), units.end());
  units.erase(std::unique(units.begin(), units.end()), units.end());
  const int n_routed = (int)units.size();
  if (shared) units.push_back(-1);
  std::vector<std::vector<int>> toks(units.size());
  for (int u = 0; u < n_routed; u++)
    for (int t = 0; t < T; t++)
      for (int j = 0; j < k; j++)
        if (ids[(size_t)t * k + j] == units[u]) {
          toks[u].push_back(t);
          break;
        }
  if (shared)
    for (int t = 0; t < T; t++) toks[n_routed].push_back(t);
  std::vector<std::vector<double>> y(units.size());
  const int nu = (int)units.size();
  if (mxfp4 == 2) {
    // NVFP4 activations: x with its per-tensor scale over the T tokens; then
    // every unit's h before h's per-tensor scale (over all of them)
    float ax = 0.0f;
    for (double v : x) ax = std::max(ax, (float)std::fabs(v));
    const NvScale sx = nv_tensor_scale(ax);
    std::vector<float> xf(x.begin(), x.end());
    for (int t = 0; t < T; t++) nv_quantize_row(xf.data() + (size_t)t * H, H, sx, nullptr, nullptr, x.data() + (size_t)t * H);
    std::vector<std::vector<double>> h(units.size());
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(std::max(threads, 1))
#endif
    for (int u = 0; u < nu; u++) {
      const uint8_t* blob = units[u] < 0 ? shared : blobs[units[u]];
      const std::vector<double> wg = weight_matrix(blob, H, I, 0, fmt), wu = weight_matrix(blob, H, I, 1, fmt);
      const int m = (int)toks[u].size();
      h[u].assign((size_t)m * I, 0.0);
      for (int i = 0; i < m; i++) {
        const double* xs = x.data() + (size_t)toks[u][i] * H;
        for (int r = 0; r < I; r++) {
          double g = 0.0, uu = 0.0;
          for (int kk = 0; kk < H; kk++) {
            g += wg[(size_t)r * H + kk] * xs[kk];
            uu += wu[(size_t)r * H + kk] * xs[kk];
          }
          h[u][(size_t)i * I + r] = silu(g) * uu;
        }
      }
    }
    double ah = 0.0;
    for (const auto& hu : h)
      for (double v : hu) ah = std::max(ah, std::fabs(v));
    const NvScale sh = nv_tensor_scale((float)ah);
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(std::max(threads, 1))
#endif
    for (int u = 0; u < nu; u++) {
      const uint8_t* blob = units[u] < 0 ? shared : blobs[units[u]];
      const std::vector<double> wd = weight_matrix(blob, H, I, 2, fmt);
      const int m = (int)toks[u].size();
      y[u].assign((size_t)m * H, 0.0);
      std::vector<float> hf(I);
      std::vector<double> hq(I);
      for (int i = 0; i < m; i++) {
        for (int r = 0; r < I; r++) hf[r] = (float)h[u][(size_t)i * I + r];
        nv_quantize_row(hf.data(), I, sh, nullptr, nullptr, hq.data());
        for (int n = 0; n < H; n++) {
          double acc = 0.0;
          for (int r = 0; r < I; r++) acc += wd[(size_t)n * I + r] * hq[r];
          y[u][(size_t)i * H + n] = acc;
        }
      }
    }
  } else {
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(std::max(threads, 1))
#endif
    for (int u = 0; u < nu; u++) {
      const int m = (int)toks[u].size();
      std::vector<double> xu((size_t)m * H);
      for (int i = 0; i < m; i++) std::copy(x.begin() + (size_t)toks[u][i] * H, x.begin() + (size_t)(toks[u][i] + 1) * H,
                                            xu.begin() + (size_t)i * H);
      y[u].assign((size_t)m * H, 0.0);
      expert_ffn(units[u] < 0 ? shared : blobs[units[u]], H, I, xu.data(), m, mxfp4, fmt, y[u].data());
    }
  }
  auto y_of = [&](int u, int t) -> const double* {
    const auto& tv = toks[u];
    const int i = (int)(std::find(tv.begin(), tv.end(), t) - tv.begin());
    return y[u].data() + (size_t)i * H;
  };
  for (int t = 0; t < T; t++)
    for (int n = 0; n < H; n++) {
      double acc = 0.0;
      for (int j = 0; j < k; j++) {
        const int e = ids[(size_t)t * k + j];
        const int u = (int)(std::lower_bound(units.begin(), units.begin() + n_routed, e) - units.begin());
        acc += w[(size_t)t * k + j] * y_of(u, t)[n];
      }
      if (shared) acc += y_of(n_routed, t)[n];
      out[(size_t)t * H + n] = acc;
      if (out_bits) out_bits[(size_t)t * H + n] = round_bf16(acc);
    }
  if (ids_out) std::copy(ids.begin(), ids.end(), ids_out);
  if (w_out) std::copy(w.begin(), w.end(), w_out);
  return bad;
}

// --- LRU ---------------------------------------------------------------------
// Per layer step, S = the distinct selected experts in ascending id; a hit
// moves the key to most recent; a miss, when full, evicts the least recent key
// not in S and takes its slot, else the lowest free slot; |S| > capacity is an
// error.  Shrink: evict from the least recent end, then move survivors in
// slots >= the new capacity, in ascending slot order, to the lowest free slots.
// Events: (kind, layer, expert, slot, from_slot) with kind 0 HIT, 1 MISS,
// 2 EVICT, 3 MOVE.

FTO_API void* fto_lru_new(int64_t capacity) {
  Lru* c = new Lru();
  c->capacity = capacity;
  return c;
}

// Decode-time next-layer prefetch (the numpy oracle's PrefetchingLRUCache):
// after each step at layer l, the experts of layer (l + 1) % n_layers that
// were selected at least once, most often first (ties to the lower id), are
// inserted, up to per_layer of them, skipping resident ones; when full, the
// victim is the least recent key neither in the step's set nor of that layer.
// Events of kind 4 (PREFETCH).
FTO_API void fto_lru_set_prefetch(void* h, int n_layers, int n_experts, int per_layer) {
  Lru& c = *static_cast<Lru*>(h);
  c.n_layers = n_layers;
  c.n_experts = n_experts;
  c.per_layer = per_layer;
  c.count.assign((size_t)n_layers * n_experts, 0);
}

FTO_API void fto_lru_prefetch_counts(void* h, int64_t* out2) {
  Lru& c = *static_cast<Lru*>(h);
  out2[0] = c.prefetches;
  out2[1] = c.prefetch_hits;
}

FTO_API void fto_lru_free(void* h) { delete static_cast<Lru*>(h); }

static int lowest_free(const Lru& c) {
  std::vector<char> used((size_t)std::max<int64_t>(c.capacity, 0), 0);
  for (const auto& kv : c.slot)
    if (kv.second < c.capacity) used[kv.second] = 1;
  for (int64_t s = 0; s < c.capacity; s++)
    if (!used[s]) return (int)s;
  return -1;
}

// events out [cap][5]; returns the number of events, or -1 when |S| > capacity
FTO_API int64_t fto_lru_step(void* h, int layer, const int32_t* experts, int n, int32_t* ev, int64_t cap) {
  Lru& c = *static_cast<Lru*>(h);
  std::vector<int> S(experts, experts + n);
  std::sort(S.begin(), S.end());
  S.erase(std::unique(S.begin(), S.end()), S.end());
  if ((int64_t)S.size() > c.capacity) return -1;
  int64_t ne = 0;
  auto emit = [&](int kind, int l, int e, int s, int from) {
    if (ne < cap) {
      int32_t* p = ev + 5 * ne;
      p[0] = kind;
      p[1] = l;
      p[2] = e;
      p[3] = s;
      p[4] = from;
    }
    ne++;
  };
  for (int e : S) {
    const std::pair<int, int> key{layer, e};
    auto it = c.slot.find(key);
    if (it != c.slot.end()) {
      c.order.remove(key);
      c.order.push_back(key);
      emit(0, layer, e, it->second, -1);
      if (c.unused.erase(key)) c.prefetch_hits++;
      continue;
    }
    int s;
    if ((int64_t)c.order.size() == c.capacity) {
      auto v = c.order.begin();
      while (v->first == layer && std::binary_search(S.begin(), S.end(), v->second)) ++v;
      const std::pair<int, int> victim = *v;
      c.order.erase(v);
      s = c.slot[victim];
      c.slot.erase(victim);
      c.unused.erase(victim);
      emit(2, victim.first, victim.second, s, -1);
    } else {
      s = lowest_free(c);
    }
    c.slot[key] = s;
    c.order.push_back(key);
    emit(1, layer, e, s, -1);
  }
  if (c.n_layers <= 0) return ne;
  for (int e : S) c.count[(size_t)layer * c.n_experts + e]++;
  if (c.per_layer <= 0) return ne;
  const int nl = (layer + 1) % c.n_layers;
  std::vector<int> cand;
  for (int e = 0; e < c.n_experts; e++)
    if (c.count[(size_t)nl * c.n_experts + e] > 0) cand.push_back(e);
  const int64_t* cnt = c.count.data() + (size_t)nl * c.n_experts;
  std::stable_sort(cand.begin(), cand.end(), [&](int a, int b) { return cnt[a] > cnt[b]; });
  int done = 0;
  for (int e : cand) {
    if (done >= c.per_layer) break;
    const std::pair<int, int> key{nl, e};
    if (c.slot.count(key)) continue;
    int s;
    if ((int64_t)c.order.size() == c.capacity) {
      auto v = c.order.begin();
      while (v != c.order.end() &&
             ((v->first == layer && std::binary_search(S.begin(), S.end(), v->second)) || v->first == nl))
        ++v;
      if (v == c.order.end()) break;
      const std::pair<int, int> victim = *v;
      c.order.erase(v);
      s = c.slot[victim];
      c.slot.erase(victim);
      c.unused.erase(victim);
      emit(2, victim.first, victim.second, s, -1);
    } else {
      s = lowest_free(c);
    }
    c.slot[key] = s;
    c.order.push_back(key);
    c.unused[key] = 1;
    c.prefetches++;
    emit(4, nl, e, s, -1);
    done++;
  }
  return ne;
}

FTO_API int64_t fto_lru_resize(void* h, int64_t capacity, int32_t* ev, int64_t cap) {
  Lru& c = *static_cast<Lru*>(h);
  int64_t ne = 0;
  auto emit = [&](int kind, int l, int e, int s, int from) {
    if (ne < cap) {
      int32_t* p = ev + 5 * ne;
      p[0] = kind;
      p[1] = l;
      p[2] = e;
      p[3] = s;
      p[4] = from;
    }
    ne++;
  };
  while ((int64_t)c.order.size() > capacity) {
    const std::pair<int, int> victim = c.order.front();
    c.order.pop_front();
    const int s = c.slot[victim];
    c.slot.erase(victim);
    c.unused.erase(victim);
    emit(2, victim.first, victim.second, s, -1);
  }
  const int64_t old = c.capacity;
  c.capacity = capacity;
  if (capacity < old) {
    std::vector<std::pair<int, std::pair<int, int>>> movers;
    for (const auto& kv : c.slot)
      if (kv.second >= capacity) movers.push_back({kv.second, kv.first});
    std::sort(movers.begin(), movers.end());
    for (const auto& mv : movers) {
      const int dst = lowest_free(c);
      c.slot[mv.second] = dst;
      emit(3, mv.second.first, mv.second.second, dst, mv.first);
    }
  }
  return ne;
}

// slot of a key (touching it as most recent) or -1
FTO_API int fto_lru_lookup(void* h, int layer, int expert) {
  Lru& c = *static_cast<Lru*>(h);
  const std::pair<int, int> key{layer, expert};
  auto it = c.slot.find(key);
  if (it == c.slot.end()) return -1;
  c.order.remove(key);
  c.order.push_back(key);
  return it->second;
}

// Decode GEMV of the allocation-free forward (ft_moe_layer_forward_noalloc):
// split-K FP4 GEMV of the selected experts, dequantising e2m1 codes with their
// UE8M0 block scales in registers.  (The context's decode path is
// ft_decode.cu.)
//
//   k_gate_up        h[pair][i] = silu(Wg[i] . x) * (Wu[i] . x)      (fp32 h)
//   k_down_combine   y[pair][n] = Wd[n] . h[pair];
//                    out[t][n] = bf16( sum_j w[t][j] y[inv[t k + j]][n]  (+ shared) )
//
// Pages: experts run on the GPU from weights held there or fetched over PCIe,
// and the partial results are summed exactly (jansverre.net, "Hvorfor er
// båndbredden viktigere enn antall kjerner?").  SwiGLU experts and the fixed
// combine order are this library's reading (see ft_moe.h).
//
// Work split.  A row of a weight matrix is split along K over `lpr` lanes
// (lpr = min(32, K/32)); lane s of a row owns the 16-byte code chunks
// c = s, s + lpr, ... (32 elements, one scale block each), so every warp load
// of codes is a coalesced 128-bit load.  The lane's activations for those
// chunks stay in registers while it walks RW rows, so each activation value
// read from shared memory serves RW weight rows.  Partial sums of a row are
// reduced across its lpr lanes by an xor butterfly: this is the split-K.
#include "ft_common.cuh"
#include "ft_kernels.h"

namespace ft {

namespace {

// Dot of one 16-byte chunk of codes (32 elements) with 32 activations held as
// 16 float pairs; returns the unscaled sum.
__device__ __forceinline__ float chunk_dot(uint4 q, const float2* xv) {
  float2 acc = make_float2(0.f, 0.f);
  const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int wv = 0; wv < 4; wv++) {
#pragma unroll
    for (int b = 0; b < 4; b++) {
      float2 wf = f16x2_to_f32x2(e2m1x2_to_f16x2(qs[wv] >> (8 * b)));
      acc = ffma2(wf, xv[wv * 4 + b], acc);
    }
  }
  return acc.x + acc.y;
}

__device__ __forceinline__ float group_sum(float v, int lpr) {
  for (int d = lpr >> 1; d >= 1; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
  return v;
}

// Tokens (and h rows) of unit u: a routed active expert or a shared expert.
struct Unit {
  int e;      // blob index in the layer (E + s for shared expert s)
  int m;      // number of tokens
  int p0;     // first permuted position (routed) or -1 (shared)
  int hbase;  // first h row
};

__device__ __forceinline__ bool unit_of(const GemvParams& p, int u, Unit& out) {
  if (u < p.max_active) {
    if (u >= *p.n_active) return false;
    int e = p.active[u];
    out.e = e;
    out.p0 = p.offs[e];
    out.m = p.offs[e + 1] - out.p0;
    out.hbase = out.p0;
  } else {
    int s = u - p.max_active;
    out.e = p.E + s;
    out.m = p.T;
    out.p0 = -1;
    out.hbase = p.T * p.k + s * p.T;
  }
  return true;
}

__device__ __forceinline__ int unit_token(const GemvParams& p, const Unit& un, int i) {
  return un.p0 >= 0 ? p.perm[un.p0 + i] / p.k : i;
}

}  // namespace

// ---------------------------------------------------------------------------
// gate/up + SwiGLU.  CTA = 8 warps; lane group of lpr lanes owns RW rows.
// Activations for MT tokens are staged in shared memory as fp32 in a
// chunk-interleaved order (index ((j*8 + v) * lpr + s) * 4 + q for element
// 32 c + 4 v + q of chunk c = s + lpr j) so that the lpr lanes of a group read
// consecutive 16-byte words.
// ---------------------------------------------------------------------------
template <int MT, int RW>
__global__ void __launch_bounds__(256) k_gate_up(GemvParams p) {
  extern __shared__ float4 xs4[];
  float* xs = reinterpret_cast<float*>(xs4);
  Unit un;
  if (!unit_of(p, blockIdx.y, un)) return;
  const uint8_t* blob = p.eptr[un.e];
  if (blob == nullptr) {
    if (threadIdx.x == 0) set_status(p.status, kStMissing);
    return;
  }
  const int H = p.H, I = p.I;
  const int lpr = H / 32 < 32 ? H / 32 : 32;
  const int G = 32 / lpr;
  const int J = H / (32 * lpr);
  const int atoms_k = (int)(pad_up(H / 32, 4) / 4);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane / lpr, sl = lane % lpr;
  const int rows_per_cta = 8 * G * RW;
  const int row0 = blockIdx.x * rows_per_cta + (warp * G + g) * RW;

  for (int tp = 0; tp < un.m; tp += MT) {
    // stage x for tokens tp .. tp+MT-1 (zeros past the end)
    __syncthreads();
    for (int idx = threadIdx.x; idx < MT * (H / 4); idx += blockDim.x) {
      int mm = idx / (H / 4);
      int k4 = idx % (H / 4);               // group of 4 consecutive elements
      int c = k4 >> 3, v = k4 & 7;          // chunk, vector in chunk
      int j = c / lpr, s = c % lpr;
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (tp + mm < un.m) {
        int t = unit_token(p, un, tp + mm);
        uint2 xv = *reinterpret_cast<const uint2*>(p.x + (size_t)t * H + k4 * 4);
        val = make_float4(bf16_bits_to_f32(xv.x & 0xffff), bf16_bits_to_f32(xv.x >> 16),
                          bf16_bits_to_f32(xv.y & 0xffff), bf16_bits_to_f32(xv.y >> 16));
      }
      xs4[(size_t)mm * (H / 4) + (j * 8 + v) * lpr + s] = val;
    }
    __syncthreads();

    float accg[RW][MT], accu[RW][MT];
#pragma unroll
    for (int r = 0; r < RW; r++)
#pragma unroll
      for (int mm = 0; mm < MT; mm++) accg[r][mm] = accu[r][mm] = 0.f;

    for (int j = 0; j < J; j++) {
      const int c = sl + lpr * j;
      float2 xv[MT][16];
#pragma unroll
      for (int mm = 0; mm < MT; mm++) {
        const float4* src = xs4 + (size_t)mm * (H / 4) + (j * 8) * lpr + sl;
#pragma unroll
        for (int v = 0; v < 8; v++) {
          float4 f = src[v * lpr];
          xv[mm][2 * v] = make_float2(f.x, f.y);
          xv[mm][2 * v + 1] = make_float2(f.z, f.w);
        }
      }
      uint4 qg[RW], qu[RW];
      uint32_t sg[RW], su[RW];
#pragma unroll
      for (int r = 0; r < RW; r++) {
        int row = row0 + r;
        if (row < I) {
          qg[r] = __ldg(reinterpret_cast<const uint4*>(blob + p.lay.wg + (size_t)row * (H / 2)) + c);
          qu[r] = __ldg(reinterpret_cast<const uint4*>(blob + p.lay.wu + (size_t)row * (H / 2)) + c);
          int64_t so = sf_word(row, c >> 2, atoms_k) + (c & 3);
          sg[r] = __ldg(blob + p.lay.wg_sf + so);
          su[r] = __ldg(blob + p.lay.wu_sf + so);
        }
      }
#pragma unroll
      for (int r = 0; r < RW; r++) {
        if (row0 + r < I) {
          float scg = ue8m0_to_f32(sg[r]), scu = ue8m0_to_f32(su[r]);
#pragma unroll
          for (int mm = 0; mm < MT; mm++) {
            accg[r][mm] = fmaf(chunk_dot(qg[r], xv[mm]), scg, accg[r][mm]);
            accu[r][mm] = fmaf(chunk_dot(qu[r], xv[mm]), scu, accu[r][mm]);
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < RW; r++) {
#pragma unroll
      for (int mm = 0; mm < MT; mm++) {
        float gs = group_sum(accg[r][mm], lpr);
        float us = group_sum(accu[r][mm], lpr);
        int row = row0 + r;
        if (sl == 0 && row < I && tp + mm < un.m) p.h[(size_t)(un.hbase + tp + mm) * I + row] = silu(gs) * us;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// down + combine.  CTA = 4 warps owns output rows [n0, n0 + rows_per_cta) for
// every token; y of every pair for those rows goes to shared memory, then the
// weighted sum over j (ascending) plus shared experts is rounded to bf16.
// ---------------------------------------------------------------------------
template <int RW>
__global__ void __launch_bounds__(128) k_down_combine(GemvParams p) {
  extern __shared__ float ys[];  // [n_pairs][rows_per_cta]
  const int H = p.H, I = p.I;
  const int lpr = I / 32 < 32 ? I / 32 : 32;
  const int G = 32 / lpr;
  const int J = I / (32 * lpr);
  const int atoms_k = (int)(pad_up(I / 32, 4) / 4);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane / lpr, sl = lane % lpr;
  const int rows_per_cta = 4 * G * RW;
  const int n0 = blockIdx.x * rows_per_cta;
  const int rl0 = (warp * G + g) * RW;   // local row of this group
  const int n_units = *p.n_active;

  for (int uu = 0; uu < n_units + p.n_shared; uu++) {
    Unit un;
    int u = uu < n_units ? uu : p.max_active + (uu - n_units);
    unit_of(p, u, un);
    const uint8_t* blob = p.eptr[un.e];
    if (blob == nullptr) {
      if (threadIdx.x == 0) set_status(p.status, kStMissing);
      continue;
    }
    for (int pi = 0; pi < un.m; pi++) {
      const float* hrow = p.h + (size_t)(un.hbase + pi) * I;
      float acc[RW];
#pragma unroll
      for (int r = 0; r < RW; r++) acc[r] = 0.f;
      for (int j = 0; j < J; j++) {
        const int c = sl + lpr * j;
        float2 hv[16];
        const float4* src = reinterpret_cast<const float4*>(hrow + c * 32);
#pragma unroll
        for (int v = 0; v < 8; v++) {
          float4 f = __ldg(src + v);
          hv[2 * v] = make_float2(f.x, f.y);
          hv[2 * v + 1] = make_float2(f.z, f.w);
        }
#pragma unroll
        for (int r = 0; r < RW; r++) {
          int n = n0 + rl0 + r;
          if (n < H) {
            uint4 q = __ldg(reinterpret_cast<const uint4*>(blob + p.lay.wd + (size_t)n * (I / 2)) + c);
            uint32_t sb = __ldg(blob + p.lay.wd_sf + sf_word(n, c >> 2, atoms_k) + (c & 3));
            acc[r] = fmaf(chunk_dot(q, hv), ue8m0_to_f32(sb), acc[r]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < RW; r++) {
        float y = group_sum(acc[r], lpr);
        if (sl == 0) ys[(size_t)(un.hbase + pi) * rows_per_cta + rl0 + r] = y;
      }
    }
  }
  __syncthreads();
  // combine: fixed order j = 0..k-1, then shared experts
  for (int idx = threadIdx.x; idx < p.T * rows_per_cta; idx += blockDim.x) {
    int t = idx / rows_per_cta, rl = idx % rows_per_cta;
    int n = n0 + rl;
    if (n >= H) continue;
    float acc = 0.f;
    for (int j = 0; j < p.k; j++) {
      int f = t * p.k + j;
      acc = fmaf(p.w[f], ys[(size_t)p.inv[f] * rows_per_cta + rl], acc);
    }
    for (int s = 0; s < p.n_shared; s++) acc += ys[(size_t)(p.T * p.k + s * p.T + t) * rows_per_cta + rl];
    __nv_bfloat16 b = __float2bfloat16_rn(acc);
    p.out[(size_t)t * H + n] = *reinterpret_cast<uint16_t*>(&b);
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
static int gu_rows_per_cta(int H, int RW) {
  int lpr = H / 32 < 32 ? H / 32 : 32;
  return 8 * (32 / lpr) * RW;
}
static int dn_rows_per_cta(int I, int RW) {
  int lpr = I / 32 < 32 ? I / 32 : 32;
  return 4 * (32 / lpr) * RW;
}

// A K of c = K/32 chunks is split over lpr = min(32, c) lanes: the xor
// butterfly of group_sum needs lpr to be a power of two, and the chunk loop
// (J = c / lpr chunks per lane) needs c to be a multiple of lpr.  So c is 4, 8,
// 16 or a multiple of 32 (K = 128, 256, 512 or a multiple of 1024).  The
// gate/up kernel stages up to 4 tokens of x as fp32 in shared memory (16 * H
// bytes), which bounds H by the 227 KB a CTA may use.
static bool gemv_k_ok(int K) {
  if (K <= 0 || K % 128) return false;
  const int c = K / 32;
  return c < 32 ? (c & (c - 1)) == 0 : c % 32 == 0;
}

bool gemv_shape_ok(int H, int I) { return gemv_k_ok(H) && gemv_k_ok(I) && (size_t)16 * H <= 227 * 1024; }

template <int MT>
static cudaError_t launch_gu_mt(const GemvParams& p, cudaStream_t s) {
  constexpr int RW = 4;
  int rows = gu_rows_per_cta(p.H, RW);
  dim3 grid((p.I + rows - 1) / rows, p.max_active + p.n_shared);
  size_t smem = (size_t)MT * p.H * sizeof(float);
  // the attribute is per device: set it on every launch (cheap, and correct
  // when several devices or host threads use the library)
  cudaError_t e = cudaFuncSetAttribute(k_gate_up<MT, RW>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_gate_up<MT, RW><<<grid, 256, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gate_up(const GemvParams& p, cudaStream_t s) {
  if (p.T <= 1) return launch_gu_mt<1>(p, s);
  if (p.T <= 2) return launch_gu_mt<2>(p, s);
  return launch_gu_mt<4>(p, s);
}

cudaError_t launch_down_combine(const GemvParams& p, cudaStream_t s) {
  constexpr int RW = 2;
  int rows = dn_rows_per_cta(p.I, RW);
  int n_pairs = p.T * p.k + p.n_shared * p.T;
  size_t smem = (size_t)n_pairs * rows * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(k_down_combine<RW>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_down_combine<RW><<<(p.H + rows - 1) / rows, 128, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace ft

// Prefill path (MXFP4 activations): scratch, the activation quantiser into
// 128-padded per-expert segments, and the weighted combine.  The grouped GEMMs
// are in ft_gemm.cu; the runtime sequences the steps.
//
//   rows:  every expert e owns padded rows [pad_offs[e], pad_offs[e+1]) of the
//          activation matrices, a multiple of 128 so that a token tile of the
//          GEMM and a scale atom never straddle two experts; its first
//          offs[e+1]-offs[e] rows hold its tokens in ascending order, the rest
//          are zero.  A shared expert owns one more segment holding all tokens.
#include "ft_common.cuh"
#include "ft_gemm.h"
#include "ft_kernels.h"
#include "ft_mx.cuh"
#include "ft_runtime.h"

namespace ft {
namespace {

__device__ __forceinline__ int segment_of(const int32_t* pad_offs, int nseg, int row) {
  int lo = 0, hi = nseg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pad_offs[mid] <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void k_shared_segments(int32_t* pad_offs, int E, int T, int n_shared) {
  if (threadIdx.x == 0)
    for (int s = 0; s < n_shared; s++) pad_offs[E + 1 + s] = pad_offs[E + s] + (int32_t)pad_up(T, 128);
}

// Warp per padded row: quantise the row's token (or zeros) per 32 values.
__global__ void __launch_bounds__(256) k_quant_x(const uint16_t* __restrict__ x, int T, int H, int E, int k,
                                                 int n_seg, const int32_t* __restrict__ pad_offs,
                                                 const int32_t* __restrict__ offs, const int32_t* __restrict__ perm,
                                                 int rows_bound, uint8_t* __restrict__ xq, uint8_t* __restrict__ xq_sf) {
  const int lane = threadIdx.x & 31;
  const int p = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (p >= rows_bound || p >= pad_offs[n_seg]) return;
  const int e = segment_of(pad_offs, n_seg, p);
  const int r = p - pad_offs[e];
  const bool shared = e >= E;
  const int count = shared ? T : offs[e + 1] - offs[e];
  const int token = r < count ? (shared ? r : perm[offs[e] + r] / k) : -1;
  const int nb = H / 32, atoms_k = H / 128;
  for (int b = lane; b < nb; b += 32) {
    uint4 q = make_uint4(0, 0, 0, 0);
    uint32_t sc = 0;
    if (token >= 0) {
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)token * H + b * 32);
      float4 v[8];
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const uint4 w = __ldg(src + i);
        v[2 * i] = make_float4(bf16_bits_to_f32(w.x & 0xffff), bf16_bits_to_f32(w.x >> 16),
                               bf16_bits_to_f32(w.y & 0xffff), bf16_bits_to_f32(w.y >> 16));
        v[2 * i + 1] = make_float4(bf16_bits_to_f32(w.z & 0xffff), bf16_bits_to_f32(w.z >> 16),
                                   bf16_bits_to_f32(w.w & 0xffff), bf16_bits_to_f32(w.w >> 16));
      }
      sc = mx_quant_block(v, q);
    }
    *reinterpret_cast<uint4*>(xq + (size_t)p * (H / 2) + b * 16) = q;
    xq_sf[sf_word(p, b >> 2, atoms_k) + (b & 3)] = (uint8_t)sc;
  }
}

// NVFP4 variant of k_quant_x: per 16 values, with the per-tensor scale of x
// from *amax (all T tokens).
__global__ void __launch_bounds__(256) k_quant_x_nv(const uint16_t* __restrict__ x, int T, int H, int E, int k,
                                                    int n_seg, const int32_t* __restrict__ pad_offs,
                                                    const int32_t* __restrict__ offs, const int32_t* __restrict__ perm,
                                                    int rows_bound, const uint32_t* __restrict__ amax,
                                                    uint8_t* __restrict__ xq, uint8_t* __restrict__ xq_sf) {
  const int lane = threadIdx.x & 31;
  const int p = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (p >= rows_bound || p >= pad_offs[n_seg]) return;
  const NvScale ts = nv_tensor_scale(*amax);
  const int e = segment_of(pad_offs, n_seg, p);
  const int r = p - pad_offs[e];
  const bool shared = e >= E;
  const int count = shared ? T : offs[e + 1] - offs[e];
  const int token = r < count ? (shared ? r : perm[offs[e] + r] / k) : -1;
  const int atoms_k = H / 64;
  for (int b = lane; b < H / 32; b += 32) {
    uint2 q0 = make_uint2(0u, 0u), q1 = q0;
    uint32_t e0 = 0, e1 = 0;
    if (token >= 0) {
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)token * H + b * 32);
      float v[2][16];
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const uint4 w = __ldg(src + i);
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
          v[i >> 1][8 * (i & 1) + 2 * j] = bf16_bits_to_f32(u[j] & 0xffff);
          v[i >> 1][8 * (i & 1) + 2 * j + 1] = bf16_bits_to_f32(u[j] >> 16);
        }
      }
      e0 = nv_quant_block16(v[0], ts, q0);
      e1 = nv_quant_block16(v[1], ts, q1);
    }
    *reinterpret_cast<uint4*>(xq + (size_t)p * (H / 2) + b * 16) = make_uint4(q0.x, q0.y, q1.x, q1.y);
    *reinterpret_cast<uint16_t*>(xq_sf + sf_word(p, b >> 1, atoms_k) + ((2 * b) & 3)) = (uint16_t)(e0 | (e1 << 8));
  }
}

// NVFP4 h: the gate/up GEMM left h in fp32 ([rows][I], padded rows) and its
// largest magnitude in *amax; quantise every padded row with that per-tensor
// scale (padding rows are zeros and give zero codes and scales).
__global__ void __launch_bounds__(256) k_quant_h_nv(const float* __restrict__ hf, int I, int T, int E, int n_seg,
                                                    const int32_t* __restrict__ pad_offs,
                                                    const int32_t* __restrict__ offs, int rows_bound,
                                                    const uint32_t* __restrict__ amax, uint8_t* __restrict__ hq,
                                                    uint8_t* __restrict__ hq_sf) {
  const int lane = threadIdx.x & 31;
  const int p = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (p >= rows_bound || p >= pad_offs[n_seg]) return;
  const NvScale ts = nv_tensor_scale(*amax);
  const int atoms_k = I / 64;
  const int e = segment_of(pad_offs, n_seg, p);
  // a padding row of the segment: its h (never stored) is zero
  const bool pad = p - pad_offs[e] >= (e >= E ? T : offs[e + 1] - offs[e]);
  for (int b = lane; b < I / 32; b += 32) {
    const float4* src = reinterpret_cast<const float4*>(hf + (size_t)p * I + b * 32);
    float v[2][16];
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const float4 f = pad ? make_float4(0.f, 0.f, 0.f, 0.f) : src[i];
      v[i >> 2][4 * (i & 3)] = f.x;
      v[i >> 2][4 * (i & 3) + 1] = f.y;
      v[i >> 2][4 * (i & 3) + 2] = f.z;
      v[i >> 2][4 * (i & 3) + 3] = f.w;
    }
    uint2 q0, q1;
    const uint32_t e0 = nv_quant_block16(v[0], ts, q0), e1 = nv_quant_block16(v[1], ts, q1);
    *reinterpret_cast<uint4*>(hq + (size_t)p * (I / 2) + b * 16) = make_uint4(q0.x, q0.y, q1.x, q1.y);
    *reinterpret_cast<uint16_t*>(hq_sf + sf_word(p, b >> 1, atoms_k) + ((2 * b) & 3)) = (uint16_t)(e0 | (e1 << 8));
  }
}

// out[t][n] = bf16( sum_j w[t][j] * y[inv[t*k+j]][n]  +  sum_s y[T*k + s*T + t][n] )
// A thread takes four consecutive n (16-byte loads of y, one 8-byte store);
// each element's sum is taken in the order above.
__global__ void __launch_bounds__(256) k_combine(const float* __restrict__ y, const float* __restrict__ w,
                                                 const int32_t* __restrict__ inv, int T, int H, int k, int n_shared,
                                                 uint16_t* __restrict__ out) {
  const int H4 = H / 4;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)T * H4) return;
  const int t = (int)(i / H4), n = 4 * (int)(i % H4);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; j++) {
    const int f = t * k + j;
    const float wf = w[f];
    const float4 v = *reinterpret_cast<const float4*>(y + (size_t)inv[f] * H + n);
    acc.x = fmaf(wf, v.x, acc.x);
    acc.y = fmaf(wf, v.y, acc.y);
    acc.z = fmaf(wf, v.z, acc.z);
    acc.w = fmaf(wf, v.w, acc.w);
  }
  for (int s = 0; s < n_shared; s++) {
    const float4 v = *reinterpret_cast<const float4*>(y + (size_t)(T * k + s * T + t) * H + n);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
  *reinterpret_cast<uint2*>(out + (size_t)t * H + n) =
      make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
}

}  // namespace

int64_t prefill_rows_bound(int T, int E, int k, int n_shared) {
  return pad_up((int64_t)T * k + 127ll * E + (int64_t)n_shared * pad_up(T, 128), 128);
}

ft_status ensure_prefill_scratch(PrefillScratch& s, const ft_model_desc& d, int max_tokens) {
  if (s.y) return FT_OK;
  const int64_t T = max_tokens, k = d.top_k, S = d.n_shared;
  s.H = d.hidden;
  s.I = d.inter;
  s.max_pairs = T * k + S * T;
  s.max_rows = prefill_rows_bound(max_tokens, d.n_experts, d.top_k, d.n_shared);
  s.fmt = d.weight_format == FT_FMT_NVFP4 ? kFmtNv : kFmtMx;
  const int blk = s.fmt == kFmtNv ? 16 : 32;  // elements per block scale
  if (cudaMalloc(&s.xq, (size_t)s.max_rows * s.H / 2) != cudaSuccess ||
      cudaMalloc(&s.xq_sf, (size_t)s.max_rows * s.H / blk) != cudaSuccess ||
      cudaMalloc(&s.hq, (size_t)s.max_rows * s.I / 2) != cudaSuccess ||
      cudaMalloc(&s.hq_sf, (size_t)s.max_rows * s.I / blk) != cudaSuccess ||
      cudaMalloc(&s.y, (size_t)s.max_pairs * s.H * sizeof(float)) != cudaSuccess ||
      (s.fmt == kFmtNv && (cudaMalloc(&s.hf, (size_t)s.max_rows * s.I * sizeof(float)) != cudaSuccess ||
                           cudaMalloc(&s.amax, 2 * sizeof(uint32_t)) != cudaSuccess))) {
    free_prefill_scratch(s);
    return FT_ERR_CUDA;
  }
  if (encode_tmap_2d(&s.map_xq, s.xq, s.H / 2, s.max_rows, s.H / 2) != FT_OK ||
      encode_tmap_2d(&s.map_hq, s.hq, s.I / 2, s.max_rows, s.I / 2) != FT_OK) {
    free_prefill_scratch(s);
    return FT_ERR_CUDA;
  }
  return FT_OK;
}

void free_prefill_scratch(PrefillScratch& s) {
  cudaFree(s.xq);
  cudaFree(s.xq_sf);
  cudaFree(s.hq);
  cudaFree(s.hq_sf);
  cudaFree(s.y);
  cudaFree(s.hf);
  cudaFree(s.amax);
  s = PrefillScratch{};
}

cudaError_t launch_shared_segments(int32_t* pad_offs, int E, int T, int n_shared, cudaStream_t st) {
  if (n_shared <= 0) return cudaSuccess;
  k_shared_segments<<<1, 32, 0, st>>>(pad_offs, E, T, n_shared);
  return cudaGetLastError();
}

cudaError_t launch_quant_x(const PrefillScratch& s, const PrefillArgs& a, cudaStream_t st) {
  const int64_t rows = prefill_rows_bound(a.T, a.E, a.k, a.n_shared);
  if (s.fmt == kFmtNv) {
    // the per-tensor scale of x: largest |x| over all T tokens
    cudaError_t e;
    if ((e = cudaMemsetAsync(s.amax, 0, 2 * sizeof(uint32_t), st)) != cudaSuccess ||
        (e = launch_amax(a.x, (int64_t)a.T * a.H, true, s.amax, st)) != cudaSuccess)
      return e;
    k_quant_x_nv<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(a.x, a.T, a.H, a.E, a.k, a.E + a.n_shared, a.pad_offs,
                                                            a.offs, a.perm, (int)rows, s.amax, s.xq, s.xq_sf);
    return cudaGetLastError();
  }
  k_quant_x<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(a.x, a.T, a.H, a.E, a.k, a.E + a.n_shared, a.pad_offs, a.offs,
                                                       a.perm, (int)rows, s.xq, s.xq_sf);
  return cudaGetLastError();
}

cudaError_t launch_quant_h(const PrefillScratch& s, const PrefillArgs& a, cudaStream_t st) {
  if (s.fmt != kFmtNv) return cudaSuccess;  // MXFP4: the gate/up epilogue wrote hq itself
  const int64_t rows = prefill_rows_bound(a.T, a.E, a.k, a.n_shared);
  k_quant_h_nv<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(s.hf, a.I, a.T, a.E, a.E + a.n_shared, a.pad_offs, a.offs,
                                                          (int)rows, s.amax + 1, s.hq, s.hq_sf);
  return cudaGetLastError();
}

static GemmArgs gemm_args(const PrefillScratch& s, const PrefillArgs& a, int mode) {
  GemmArgs g{};
  g.K = mode == 0 ? a.H : a.I;
  g.M = mode == 0 ? a.I : a.H;
  g.n_tiles_max = (int)(prefill_rows_bound(a.T, a.E, a.k, a.n_shared) / kGemmBN);
  g.n_segments = a.E + a.n_shared;
  g.pad_offs = a.pad_offs;
  g.offs = a.offs;
  g.T = a.T;
  g.k = a.k;
  g.E = a.E;
  g.blob_stride = a.lay.stride;
  g.sfa_off[0] = mode == 0 ? a.lay.wg_sf : a.lay.wd_sf;
  g.sfa_off[1] = mode == 0 ? a.lay.wu_sf : a.lay.wd_sf;
  g.pool = a.pool;
  g.sfb = mode == 0 ? s.xq_sf : s.hq_sf;
  g.mode = mode;
  g.fmt = s.fmt;
  if (s.fmt == kFmtNv) {
    g.ts_off = a.lay.ts;
    g.amax_in = s.amax + (mode == 0 ? 0 : 1);  // x for gate/up, h for down
    g.amax_out = s.amax + 1;
    g.hf = s.hf;
  }
  g.hq = s.hq;
  g.hq_sf = s.hq_sf;
  g.y = s.y;
  g.status = a.status;
  return g;
}

cudaError_t launch_prefill_gemm(const PrefillScratch& s, const PrefillArgs& a, int mode, cudaStream_t st) {
  GemmMaps m{};
  const int n_blobs = a.E + a.n_shared;
  const uint64_t stride = (uint64_t)a.lay.stride;
  if (mode == 0) {
    if (encode_tmap_3d(&m.a[0], a.pool + a.lay.wg, a.H / 2, a.I, n_blobs, a.H / 2, stride) != FT_OK ||
        encode_tmap_3d(&m.a[1], a.pool + a.lay.wu, a.H / 2, a.I, n_blobs, a.H / 2, stride) != FT_OK)
      return cudaErrorInvalidValue;
    m.b = s.map_xq;
  } else {
    if (encode_tmap_3d(&m.a[0], a.pool + a.lay.wd, a.I / 2, a.H, n_blobs, a.I / 2, stride) != FT_OK)
      return cudaErrorInvalidValue;
    m.a[1] = m.a[0];
    m.b = s.map_hq;
  }
  return launch_gemm(gemm_args(s, a, mode), m, st);
}

cudaError_t launch_prefill_combine(const PrefillScratch& s, const PrefillArgs& a, cudaStream_t st) {
  const int64_t n = (int64_t)a.T * (a.H / 4);  // H % 128 == 0: whole groups of four
  k_combine<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(s.y, a.w, a.inv, a.T, a.H, a.k, a.n_shared, a.out);
  return cudaGetLastError();
}

}  // namespace ft

// Device filler for the seeded expert blobs of synth/gen.py: the same
// counter-based generator (splitmix64 finaliser over a counter) producing the
// same bytes, so multi-GB pools need not be generated on the host.  Holds no
// arithmetic of the MoE method.
#include <cstdint>
#include <cuda_runtime.h>

namespace {
__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__device__ __forceinline__ uint64_t stream_base(uint64_t seed, uint64_t stream) {
  return mix64(seed ^ (stream * 0xD1B54A32D192ED03ull));
}
__device__ __forceinline__ uint32_t draw_code(uint32_t b) {
  const uint32_t cum[8] = {12, 35, 56, 74, 97, 116, 125, 128};
  uint32_t u = b & 0x7f, mag = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) mag += (cum[i] <= u) ? 1u : 0u;
  return (((b >> 7) & 1u) << 3) | mag;
}

__global__ void k_fill(uint8_t* dst, int64_t stride, int64_t codes_end, int64_t used, uint64_t seed, int layer,
                       int expert0, int n) {
  const int64_t code_words = (codes_end + 3) / 4;
  const int64_t sc_bytes = used - codes_end;
  const int64_t sc_words = (sc_bytes + 7) / 8;
  const int64_t pad_bytes = stride - used;
  const int64_t per_blob = code_words + sc_words + pad_bytes;
  const int64_t total = per_blob * n;
  for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < total; g += (int64_t)gridDim.x * blockDim.x) {
    int bi = (int)(g / per_blob);
    int64_t i = g % per_blob;
    int expert = expert0 + bi;
    uint8_t* blob = dst + (int64_t)bi * stride;
    uint64_t key_hi = ((uint64_t)(layer & 0xffff) << 16 | (uint64_t)(expert & 0xffff)) << 8;
    if (i < code_words) {
      uint64_t w = mix64(stream_base(seed, key_hi | 0) + (uint64_t)(i + 1) * 0x9E3779B97F4A7C15ull);
#pragma unroll
      for (int q = 0; q < 4; q++) {
        int64_t byte = i * 4 + q;
        if (byte < codes_end) {
          uint32_t f = (uint32_t)(w >> (16 * q)) & 0xffffu;
          blob[byte] = (uint8_t)(draw_code(f & 0xff) | (draw_code(f >> 8) << 4));
        }
      }
    } else if (i < code_words + sc_words) {
      int64_t wi = i - code_words;
      uint64_t w = mix64(stream_base(seed, key_hi | 1) + (uint64_t)(wi + 1) * 0x9E3779B97F4A7C15ull);
#pragma unroll
      for (int q = 0; q < 8; q++) {
        int64_t byte = wi * 8 + q;
        if (byte < sc_bytes) {
          uint32_t b = (uint32_t)(w >> (8 * q)) & 0xffu;
          blob[codes_end + byte] = (uint8_t)(b < 64 ? 119 : (b >= 192 ? 121 : 120));
        }
      }
    } else {
      blob[used + (i - code_words - sc_words)] = 0;
    }
  }
}
}  // namespace

// BF16 and NVFP4 blobs of synth/gen.py (expert_blob_bf16, expert_blob_nvfp4):
// the same streams and draws.
__device__ __forceinline__ uint32_t bf16_draw(uint32_t f) {
  // binade of N(0, 0.02) out of 256 (BF16_BINADE_COUNTS), lowest binade 2^-14
  const uint32_t cum[11] = {1, 2, 4, 9, 19, 39, 77, 144, 225, 255, 256};
  uint32_t u = f & 0xffu, binade = 0;
#pragma unroll
  for (int i = 0; i < 11; i++) binade += (cum[i] <= u) ? 1u : 0u;
  const uint32_t frac = (f >> 8) & 0x7fu, sign = (f >> 15) & 1u;
  return (sign << 15) | ((binade + 113u) << 7) | frac;
}

__global__ void k_fill_bf16(uint8_t* dst, int64_t stride, int64_t used, uint64_t seed, int layer, int expert0, int n) {
  const int64_t words = (used / 2 + 3) / 4;  // four bf16 per 64-bit draw
  const int64_t pad_bytes = stride - used;
  const int64_t per_blob = words + pad_bytes;
  const int64_t total = per_blob * n;
  for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < total; g += (int64_t)gridDim.x * blockDim.x) {
    const int bi = (int)(g / per_blob);
    const int64_t i = g % per_blob;
    uint8_t* blob = dst + (int64_t)bi * stride;
    const uint64_t key = (((uint64_t)(layer & 0xffff) << 16 | (uint64_t)((expert0 + bi) & 0xffff)) << 8) | 2;
    if (i < words) {
      const uint64_t w = mix64(stream_base(seed, key) + (uint64_t)(i + 1) * 0x9E3779B97F4A7C15ull);
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const int64_t e = i * 4 + q;
        if (2 * e < used) {
          const uint32_t b = bf16_draw((uint32_t)(w >> (16 * q)) & 0xffffu);
          blob[2 * e] = (uint8_t)(b & 0xff);
          blob[2 * e + 1] = (uint8_t)(b >> 8);
        }
      }
    } else {
      blob[used + (i - words)] = 0;
    }
  }
}

// NVFP4: codes as the MXFP4 filler (region 0), E4M3 block scales uniform over
// 0x72..0x75 (region 3), then the three matrix scales and zeros.
__global__ void k_fill_nv(uint8_t* dst, int64_t stride, int64_t codes_end, int64_t ts_off, uint64_t seed, int layer,
                          int expert0, int n) {
  const int64_t code_words = (codes_end + 3) / 4;
  const int64_t sc_bytes = ts_off - codes_end;
  const int64_t sc_words = (sc_bytes + 7) / 8;
  const int64_t tail = stride - ts_off;
  const int64_t per_blob = code_words + sc_words + tail;
  const int64_t total = per_blob * n;
  const float tsv[3] = {0.875f * 6.103515625e-05f, 1.125f * 6.103515625e-05f, 1.375f * 6.103515625e-05f};
  for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < total; g += (int64_t)gridDim.x * blockDim.x) {
    const int bi = (int)(g / per_blob);
    const int64_t i = g % per_blob;
    uint8_t* blob = dst + (int64_t)bi * stride;
    const uint64_t key_hi = ((uint64_t)(layer & 0xffff) << 16 | (uint64_t)((expert0 + bi) & 0xffff)) << 8;
    if (i < code_words) {
      const uint64_t w = mix64(stream_base(seed, key_hi | 0) + (uint64_t)(i + 1) * 0x9E3779B97F4A7C15ull);
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const int64_t byte = i * 4 + q;
        if (byte < codes_end) {
          const uint32_t f = (uint32_t)(w >> (16 * q)) & 0xffffu;
          blob[byte] = (uint8_t)(draw_code(f & 0xff) | (draw_code(f >> 8) << 4));
        }
      }
    } else if (i < code_words + sc_words) {
      const int64_t wi = i - code_words;
      const uint64_t w = mix64(stream_base(seed, key_hi | 3) + (uint64_t)(wi + 1) * 0x9E3779B97F4A7C15ull);
#pragma unroll
      for (int q = 0; q < 8; q++) {
        const int64_t byte = wi * 8 + q;
        if (byte < sc_bytes) blob[codes_end + byte] = (uint8_t)(0x72u + ((uint32_t)(w >> (8 * q)) & 3u));
      }
    } else {
      const int64_t j = i - code_words - sc_words;  // byte of the tail
      uint8_t v = 0;
      if (j < 12) {
        const float f = tsv[j / 4];
        v = (uint8_t)((__float_as_uint(f) >> (8 * (j % 4))) & 0xffu);
      }
      blob[ts_off + j] = v;
    }
  }
}

// Fill n blobs (experts expert0 .. expert0+n-1 of `layer`) at dst + i*stride.
extern "C" __attribute__((visibility("default"))) int ftsynth_fill_blobs(void* dst, int64_t stride, int64_t codes_end, int64_t used, uint64_t seed,
                                  int32_t layer, int32_t expert0, int32_t n, void* stream) {
  if (n <= 0) return 0;
  k_fill<<<148 * 8, 256, 0, (cudaStream_t)stream>>>((uint8_t*)dst, stride, codes_end, used, seed, layer, expert0, n);
  return (int)cudaGetLastError();
}

// BF16 blobs (used = 6*H*I bytes of weights) or NVFP4 blobs (codes_end bytes
// of codes, matrix scales at ts_off).
extern "C" __attribute__((visibility("default"))) int ftsynth_fill_blobs_bf16(void* dst, int64_t stride, int64_t used,
                                                                             uint64_t seed, int32_t layer,
                                                                             int32_t expert0, int32_t n, void* stream) {
  if (n <= 0) return 0;
  k_fill_bf16<<<148 * 8, 256, 0, (cudaStream_t)stream>>>((uint8_t*)dst, stride, used, seed, layer, expert0, n);
  return (int)cudaGetLastError();
}

extern "C" __attribute__((visibility("default"))) int ftsynth_fill_blobs_nvfp4(void* dst, int64_t stride, int64_t codes_end,
                                                                              int64_t ts_off, uint64_t seed, int32_t layer,
                                                                              int32_t expert0, int32_t n, void* stream) {
  if (n <= 0) return 0;
  k_fill_nv<<<148 * 8, 256, 0, (cudaStream_t)stream>>>((uint8_t*)dst, stride, codes_end, ts_off, seed, layer, expert0,
                                                       n);
  return (int)cudaGetLastError();
}

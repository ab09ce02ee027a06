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

// Fill n blobs (experts expert0 .. expert0+n-1 of `layer`) at dst + i*stride.
extern "C" __attribute__((visibility("default"))) int ftsynth_fill_blobs(void* dst, int64_t stride, int64_t codes_end, int64_t used, uint64_t seed,
                                  int32_t layer, int32_t expert0, int32_t n, void* stream) {
  if (n <= 0) return 0;
  k_fill<<<148 * 8, 256, 0, (cudaStream_t)stream>>>((uint8_t*)dst, stride, codes_end, used, seed, layer, expert0, n);
  return (int)cudaGetLastError();
}

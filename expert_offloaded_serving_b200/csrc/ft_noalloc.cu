// ft_moe_layer_forward_noalloc: the decode forward for callers that must not
// allocate device memory.
//
// Some callers cannot call cudaMalloc: a serving process whose device memory
// is owned entirely by another allocator (for example a framework's caching
// allocator that has reserved the whole budget), or a latency-critical path
// that cannot accept the implicit device-wide synchronisation cudaMalloc and
// cudaFree may cause.  This entry point needs no context and allocates
// nothing: its scratch (routing ids and weights, the permutation, the blob
// pointer table and the fp32 SwiGLU activations) lives in one file-scope
// __device__ array of kNoAllocScratchBytes, which every GPU that loads the
// library holds until the process exits.  It computes what the decode path of
// ft_moe_layer_forward computes on a resident layer pool, with the
// context-free kernels: the router GEMV, top-k and permutation of
// ft_route.cu, then the split-K GEMVs of ft_gemv.cu (launch_gate_up,
// launch_down_combine).  Those GEMVs take fewer shapes than the context's
// decode kernels (see gemv_shape_ok) and round differently (fp32 x and h, no
// f16 re-encoding), so the two paths agree within the output tolerance, not
// bit for bit.
#include <cstdio>
#include <mutex>

#include "ft_common.cuh"
#include "ft_kernels.h"
#include "ft_runtime.h"

namespace {

constexpr size_t kNoAllocScratchBytes = FT_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
unsigned char* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device.  The array's name
// is only a host-side stand-in in host code, so the address is looked up once
// per device with that device current.
ft_status scratch_for_current_device(unsigned char** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    ft::set_last_error("no usable current CUDA device");
    return FT_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char buf[256];
      snprintf(buf, sizeof buf, "cudaGetSymbolAddress of the scratch array failed: %s", cudaGetErrorString(e));
      ft::set_last_error(buf);
      return FT_ERR_CUDA;
    }
    g_scratch_ptr[dev] = (unsigned char*)p;
  }
  *out = g_scratch_ptr[dev];
  return FT_OK;
}

__global__ void k_fill_eptr(const uint8_t* base, int64_t stride, int n, const uint8_t** eptr) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) eptr[i] = base + (int64_t)i * stride;
}

ft_status bad(const char* msg) {
  ft::set_last_error(msg);
  return FT_ERR_INVALID;
}

}  // namespace

extern "C" ft_status ft_moe_layer_forward_noalloc(int32_t hidden, int32_t inter, int32_t n_experts, int32_t top_k,
                                                  int32_t n_shared, const void* layer_pool, const void* x, int64_t T,
                                                  const float* router_w, const float* logits_override, void* out,
                                                  uint32_t flags, int32_t* status, void* stream) {
  const int H = hidden, I = inter, E = n_experts, k = top_k, S = n_shared;
  if (!layer_pool || !out || (!x && T > 0)) return bad("NULL argument");
  if (H <= 0 || H % 128 || I <= 0 || I % 128) return bad("hidden and inter must be positive multiples of 128");
  if (!ft::gemv_shape_ok(H, I))
    return bad("hidden and inter must each be 128, 256, 512 or a multiple of 1024, and hidden at most 14336");
  if (E <= 0 || E > 1024 || k <= 0 || k > 16 || k > E || S < 0 || S > 1) return bad("bad expert counts");
  if (T < 0 || T > ft::kDecodeMaxTokens) return bad("T outside [0, 16] (decode path only)");
  if (flags & FT_ACT_MXFP4) return bad("only the decode (bf16-activation) path has a no-alloc form");
  if (!logits_override && !router_w) return bad("need router_w or logits_override");
  if (x == out) return bad("out must not alias x");
  if (!ft::aligned16(layer_pool) || !ft::aligned16(x) || !ft::aligned16(out) || !ft::aligned16(router_w) ||
      !ft::aligned16(logits_override))
    return bad("layer_pool, x, out, router_w and logits must start on a 16-byte boundary");
  if (T == 0) return FT_OK;
  const int Ti = (int)T;

  // carve the scratch array
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += (bytes + 255) / 256 * 256;
    return o;
  };
  const size_t o_status = take(sizeof(int));
  const size_t o_logits = logits_override ? 0 : take((size_t)Ti * E * sizeof(float));
  const size_t o_ids = take((size_t)Ti * k * sizeof(int32_t));
  const size_t o_w = take((size_t)Ti * k * sizeof(float));
  const size_t o_offs = take((size_t)(E + 1) * sizeof(int32_t));
  const size_t o_perm = take((size_t)Ti * k * sizeof(int32_t));
  const size_t o_inv = take((size_t)Ti * k * sizeof(int32_t));
  const size_t o_active = take((size_t)E * sizeof(int32_t));
  const size_t o_nact = take(sizeof(int32_t));
  const size_t o_eptr = take((size_t)(E + S) * sizeof(void*));
  const size_t o_h = take((size_t)(Ti * k + S * Ti) * I * sizeof(float));
  if (off > kNoAllocScratchBytes) {
    char buf[256];
    snprintf(buf, sizeof buf, "this call needs %zu bytes of scratch, above the no-alloc maximum of %zu bytes", off,
             kNoAllocScratchBytes);
    ft::set_last_error(buf);
    return FT_ERR_INVALID;
  }
  unsigned char* base = nullptr;
  ft_status st = scratch_for_current_device(&base);
  if (st != FT_OK) return st;

  cudaStream_t s = (cudaStream_t)stream;
  int* st_word = status ? status : (int*)(base + o_status);
  auto cu = [](cudaError_t e) {
    if (e == cudaSuccess) return FT_OK;
    ft::set_last_error(cudaGetErrorString(e));
    return FT_ERR_CUDA;
  };
  if (!status && (st = cu(cudaMemsetAsync(st_word, 0, sizeof(int), s))) != FT_OK) return st;

  const ft::BlobLayout lay = ft::blob_layout(H, I);
  const uint8_t** eptr = (const uint8_t**)(base + o_eptr);
  k_fill_eptr<<<(E + S + 255) / 256, 256, 0, s>>>((const uint8_t*)layer_pool, lay.stride, E + S, eptr);
  if ((st = cu(cudaGetLastError())) != FT_OK) return st;

  const float* logits = logits_override;
  if (!logits) {
    float* lg = (float*)(base + o_logits);
    if ((st = cu(ft::launch_router_logits((const uint16_t*)x, router_w, Ti, H, E, lg, s))) != FT_OK) return st;
    logits = lg;
  }
  int32_t* ids = (int32_t*)(base + o_ids);
  float* w = (float*)(base + o_w);
  int32_t* offs = (int32_t*)(base + o_offs);
  int32_t* perm = (int32_t*)(base + o_perm);
  int32_t* inv = (int32_t*)(base + o_inv);
  int32_t* active = (int32_t*)(base + o_active);
  int32_t* nact = (int32_t*)(base + o_nact);
  if ((st = cu(ft::launch_topk(logits, Ti, E, k, (flags & FT_ROUTE_RENORM) ? 1 : 0, ids, w, st_word, s))) != FT_OK)
    return st;
  if ((st = cu(ft::launch_permute(ids, Ti * k, E, offs, perm, inv, active, nact, nullptr, st_word, s))) != FT_OK)
    return st;

  ft::GemvParams p{};
  p.x = (const uint16_t*)x;
  p.T = Ti;
  p.H = H;
  p.I = I;
  p.E = E;
  p.k = k;
  p.n_shared = S;
  p.max_active = Ti * k < E ? Ti * k : E;
  p.offs = offs;
  p.perm = perm;
  p.inv = inv;
  p.w = w;
  p.active = active;
  p.n_active = nact;
  p.eptr = eptr;
  p.lay = lay;
  p.h = (float*)(base + o_h);
  p.out = (uint16_t*)out;
  p.status = st_word;
  if ((st = cu(ft::launch_gate_up(p, s))) != FT_OK) return st;
  return cu(ft::launch_down_combine(p, s));
}

// Host runtime and C ABI of libftmoe.so: context, scratch, global LRU expert
// cache over a CUDA virtual-memory slot arena, pinned host pool, miss fetch,
// prefill double-buffered prefetch, elastic resize, layer orchestration.
//
// Pages: experts that are not in VRAM are fetched over PCIe (jansverre.net,
// "Hva er FreeToken?"); decoding uses one global LRU cache across the MoE
// layers instead of pinning experts at start-up, and prefill streams the next
// layer pack while the GPU works on the current one (jansverre.net, "Hvorfor
// er båndbredden viktigere enn antall kjerner?"); the shared LRU exploits the
// expert-path overlap of adjacent tokens (aipolix.com, paragraph on
// semantic-aware caching); the GPU expert cache is resized without restarting
// the engine or reloading the host-resident pool (aipolix.com, paragraph on
// elastic memory management).
#include <cuda.h>  // driver types only; entry points come from cudaGetDriverEntryPoint
#include <nvtx3/nvToolsExt.h>  // header-only; inert unless a profiler attaches

#include <algorithm>
#include <chrono>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <list>
#include <string>
#include <thread>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "ft_common.cuh"
#include "ft_decode.h"
#include "ft_kernels.h"
#include "ft_runtime.h"

using namespace ft;

// ---------------------------------------------------------------------------
// host-side ranges for NVTX-aware profilers (ncu --nvtx, nsys); without one
// attached the calls return at once
// ---------------------------------------------------------------------------
namespace {
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace

// ---------------------------------------------------------------------------
// errors
// ---------------------------------------------------------------------------
static thread_local std::string g_err;

static ft_status fail(ft_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

#define CUDA_TRY(expr)                                                                         \
  do {                                                                                         \
    cudaError_t e_ = (expr);                                                                   \
    if (e_ != cudaSuccess) return fail(FT_ERR_CUDA, "%s: %s (%s:%d)", #expr, cudaGetErrorString(e_), __FILE__, __LINE__); \
  } while (0)

#define CU_TRY(expr)                                                                           \
  do {                                                                                         \
    CUresult r_ = (expr);                                                                      \
    if (r_ != CUDA_SUCCESS) return fail(FT_ERR_CUDA, "%s: CUresult %d (%s:%d)", #expr, (int)r_, __FILE__, __LINE__); \
  } while (0)

extern "C" const char* ft_last_error(void) { return g_err.c_str(); }

void ft::set_last_error(const char* msg) { g_err = msg; }

// ---------------------------------------------------------------------------
// driver API entry points (no link-time dependency on libcuda)
// ---------------------------------------------------------------------------
namespace {
struct Drv {
  CUresult (*memAddressReserve)(CUdeviceptr*, size_t, size_t, CUdeviceptr, unsigned long long) = nullptr;
  CUresult (*memAddressFree)(CUdeviceptr, size_t) = nullptr;
  CUresult (*memCreate)(CUmemGenericAllocationHandle*, size_t, const CUmemAllocationProp*, unsigned long long) = nullptr;
  CUresult (*memRelease)(CUmemGenericAllocationHandle) = nullptr;
  CUresult (*memMap)(CUdeviceptr, size_t, size_t, CUmemGenericAllocationHandle, unsigned long long) = nullptr;
  CUresult (*memUnmap)(CUdeviceptr, size_t) = nullptr;
  CUresult (*memSetAccess)(CUdeviceptr, size_t, const CUmemAccessDesc*, size_t) = nullptr;
  CUresult (*memGetAllocationGranularity)(size_t*, const CUmemAllocationProp*, CUmemAllocationGranularity_flags) = nullptr;
  bool ok = false;
};

ft_status load_driver(Drv& d) {
  if (d.ok) return FT_OK;
  struct Ent {
    const char* name;
    void** fn;
  } ents[] = {{"cuMemAddressReserve", (void**)&d.memAddressReserve},
              {"cuMemAddressFree", (void**)&d.memAddressFree},
              {"cuMemCreate", (void**)&d.memCreate},
              {"cuMemRelease", (void**)&d.memRelease},
              {"cuMemMap", (void**)&d.memMap},
              {"cuMemUnmap", (void**)&d.memUnmap},
              {"cuMemSetAccess", (void**)&d.memSetAccess},
              {"cuMemGetAllocationGranularity", (void**)&d.memGetAllocationGranularity}};
  for (auto& e : ents) {
    cudaDriverEntryPointQueryResult q;
    cudaError_t err = cudaGetDriverEntryPoint(e.name, e.fn, cudaEnableDefault, &q);
    if (err != cudaSuccess || q != cudaDriverEntryPointSuccess || *e.fn == nullptr)
      return fail(FT_ERR_CUDA, "driver entry point %s unavailable", e.name);
  }
  d.ok = true;
  return FT_OK;
}
}  // namespace

// ---------------------------------------------------------------------------
// global LRU over (layer, expert) keys
// ---------------------------------------------------------------------------
namespace {
struct Lru {
  // most recent at the back
  std::list<int64_t> order;
  std::unordered_map<int64_t, std::pair<int32_t, std::list<int64_t>::iterator>> map;  // key -> (slot, pos)
  std::vector<char> slot_used;
  int64_t capacity = 0;

  int32_t lowest_free() const {
    for (int64_t s = 0; s < capacity; s++)
      if (!slot_used[s]) return (int32_t)s;
    return -1;
  }
  void set_capacity(int64_t c) {
    capacity = c;
    if ((int64_t)slot_used.size() < c) slot_used.resize(c, 0);
  }
};
}  // namespace

// ---------------------------------------------------------------------------
// context
// ---------------------------------------------------------------------------
struct ft_ctx {
  ft_model_desc d{};
  BlobLayout lay{};
  int64_t stride = 0;
  int n_blobs = 0;  // E + n_shared per layer
  int device = 0;
  int max_tokens = 0;

  std::vector<const uint8_t*> host_layers;
  std::vector<void*> registered;  // host ranges we pinned with cudaHostRegister
  std::vector<const uint8_t*> resident;

  cudaStream_t copy_stream = nullptr;
  cudaStream_t last_stream = nullptr;

  // device scratch
  int* d_status = nullptr;
  float* d_logits = nullptr;
  int32_t* d_ids = nullptr;
  float* d_w = nullptr;
  int32_t* d_offs = nullptr;
  int32_t* d_perm = nullptr;
  int32_t* d_inv = nullptr;
  int32_t* d_active = nullptr;
  int32_t* d_nact = nullptr;
  int32_t* d_pad_offs = nullptr;
  float* d_h = nullptr;
  float* d_y = nullptr;        // decode y [(T*k + S*T)][H]
  Route* d_routes = nullptr;   // decode routing records [L]
  int* d_counters = nullptr;   // decode combine counters [(H/128) * 8]
  uint16_t* d_xbuf[2] = {nullptr, nullptr};  // stack forward ping-pong [T][H]
  int* d_sync = nullptr;       // persistent stack kernel counters [L][sync_stride]
  int sync_stride = 0;
  int* d_flag = nullptr;       // a device flag nothing sets (failure injection)
  uint32_t* d_qamax = nullptr; // ft_quantize_nvfp4: largest |x| (fp32 bits)
  uint64_t* d_tagged = nullptr;    // persistent kernels, T <= 2: tagged h, then tagged x
  uint64_t* d_h_tagged = nullptr;  // [T*k + S*T][I] words
  uint64_t* d_x_tagged = nullptr;  // [T][H/2] words (dataflow kernel)
  int64_t tagged_words = 0;
  uint32_t* d_epoch = nullptr;     // launch counter for those tags
  uint64_t* timeline = nullptr;    // dataflow kernel phase stamps (caller's device buffer) or NULL
  int64_t timeline_words = 0;

  // failure injection
  double host_wait_s = kHostWaitSeconds;  // limit of the bounded host waits
  int64_t fail_copy_in = 0;               // the n-th next expert copy fails (0: off)
  int decode_max_t = 0;

  // pinned host scratch
  int32_t* h_ids = nullptr;
  int* h_status = nullptr;
  cudaEvent_t ev_ids = nullptr;

  // pointer tables
  const uint8_t** d_eptr_res = nullptr;    // [L][n_blobs]
  const uint8_t** h_eptr_cache = nullptr;  // pinned [L][n_blobs]
  const uint8_t** d_eptr_cache = nullptr;  // [L][n_blobs]

  // cache arena
  Drv drv;
  CUdeviceptr va = 0;
  size_t va_size = 0;
  size_t chunk = 0;
  std::vector<CUmemGenericAllocationHandle> chunks;
  Lru lru;
  bool cache_on = false;
  uint8_t* d_shared = nullptr;  // [L][n_shared] blobs for non-resident layers
  std::vector<ft_cache_event> trace;
  int64_t trace_dropped = 0;  // events not recorded because the trace was full
  ft_cache_stats stats{};
  // Timing of one cache step with misses: ref precedes everything of the step
  // (recorded with the routed ids the host waited for), c0 / c1 bracket the
  // step's copies on the copy stream, h0 / h1 the resident experts' kernels
  // that run while the copies are in flight (NULL without such kernels).
  struct StepTiming {
    cudaEvent_t ref, c0, c1, h0, h1;
  };
  std::vector<StepTiming> copy_timing;   // steps whose events are still in flight
  std::vector<cudaEvent_t> spare_events;  // finished timing events, reused
  std::vector<cudaEvent_t> miss_events;   // one per miss copy of the current step (no timing)
  std::vector<cudaEvent_t> spare_miss_events;
  // next-layer prefetch
  int prefetch_per_layer = 0;
  std::vector<int64_t> sel_count;                     // [L][E] steps whose set held the expert
  std::unordered_map<int64_t, cudaEvent_t> pending;   // prefetched keys whose copy may be in flight
  std::unordered_set<int64_t> unused_prefetch;        // prefetched keys not hit yet

  // prefill staging
  uint8_t* d_stage[2] = {nullptr, nullptr};
  const uint8_t** d_eptr_stage[2] = {nullptr, nullptr};
  int stage_layer[2] = {-1, -1};
  cudaEvent_t ev_landed[2] = {nullptr, nullptr};
  cudaEvent_t ev_done[2] = {nullptr, nullptr};
  int64_t prefetch_bytes = 0;

  // prefill scratch (allocated on first use)
  PrefillScratch pf{};

  // per-kernel timing
  bool timing = false;
  std::vector<std::pair<int, std::pair<cudaEvent_t, cudaEvent_t>>> tmarks;  // eager (class, (start, stop))
  std::vector<std::pair<int, std::pair<cudaEvent_t, cudaEvent_t>>> gmarks;  // recorded inside stream capture
  double tms[FT_K_COUNT] = {0};
  int64_t tlaunch[FT_K_COUNT] = {0};
};

// Bracket one launch with events when timing is on (and the stream is not capturing).
struct KTimer {
  ft_ctx* c;
  int cls;
  cudaStream_t s;
  cudaEvent_t a = nullptr, b = nullptr;
  bool captured = false;
  KTimer(ft_ctx* c_, int cls_, cudaStream_t s_) : c(c_), cls(cls_), s(s_) {
    if (!c->timing) return;
    cudaStreamCaptureStatus cs;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return;
    captured = cs != cudaStreamCaptureStatusNone;
    cudaEventCreate(&a);
    cudaEventCreate(&b);
    // under capture only an external record becomes a graph node that records
    cudaEventRecordWithFlags(a, s, captured ? cudaEventRecordExternal : cudaEventRecordDefault);
  }
  ~KTimer() {
    if (!a) return;
    cudaEventRecordWithFlags(b, s, captured ? cudaEventRecordExternal : cudaEventRecordDefault);
    (captured ? c->gmarks : c->tmarks).push_back({cls, {a, b}});
  }
};

static ft_status check_desc(const ft_model_desc* d) {
  if (!d) return fail(FT_ERR_INVALID, "desc is NULL");
  if (d->hidden <= 0 || d->hidden % 128) return fail(FT_ERR_INVALID, "hidden %d not a positive multiple of 128", d->hidden);
  if (d->inter <= 0 || d->inter % 128) return fail(FT_ERR_INVALID, "inter %d not a positive multiple of 128", d->inter);
  if (d->n_experts <= 0 || d->n_experts > 1024) return fail(FT_ERR_INVALID, "n_experts %d not in [1, 1024]", d->n_experts);
  if (d->top_k <= 0 || d->top_k > 16 || d->top_k > d->n_experts) return fail(FT_ERR_INVALID, "top_k %d invalid", d->top_k);
  if (d->n_layers <= 0) return fail(FT_ERR_INVALID, "n_layers %d", d->n_layers);
  if (d->n_shared < 0 || d->n_shared > 1) return fail(FT_ERR_INVALID, "n_shared %d not 0 or 1", d->n_shared);
  if (d->cache_budget_bytes < 0) return fail(FT_ERR_INVALID, "negative cache budget");
  if (d->max_tokens <= 0) return fail(FT_ERR_INVALID, "max_tokens %d", d->max_tokens);
  if (d->weight_format < FT_FMT_MXFP4 || d->weight_format > FT_FMT_BF16)
    return fail(FT_ERR_INVALID, "weight_format %d is not FT_FMT_MXFP4, FT_FMT_NVFP4 or FT_FMT_BF16", d->weight_format);
  return FT_OK;
}

extern "C" int64_t ft_blob_stride(int32_t hidden, int32_t inter) {
  if (hidden <= 0 || inter <= 0 || hidden % 32 || inter % 32) return -1;
  return blob_layout(hidden, inter).stride;
}

extern "C" ft_status ft_blob_layout_format(int32_t hidden, int32_t inter, int32_t fmt, int64_t out[9]) {
  if (!out || hidden <= 0 || inter <= 0 || hidden % 32 || inter % 32) return fail(FT_ERR_INVALID, "bad shape");
  if (fmt < FT_FMT_MXFP4 || fmt > FT_FMT_BF16) return fail(FT_ERR_INVALID, "bad weight format %d", fmt);
  BlobLayout b = blob_layout(hidden, inter, fmt);
  int64_t v[9] = {b.wg, b.wu, b.wd, b.wg_sf, b.wu_sf, b.wd_sf, b.used, b.stride, b.ts};
  memcpy(out, v, sizeof v);
  return FT_OK;
}

extern "C" ft_status ft_blob_layout(int32_t hidden, int32_t inter, int64_t out[8]) {
  if (!out || hidden <= 0 || inter <= 0 || hidden % 32 || inter % 32) return fail(FT_ERR_INVALID, "bad shape");
  BlobLayout b = blob_layout(hidden, inter);
  int64_t v[8] = {b.wg, b.wu, b.wd, b.wg_sf, b.wu_sf, b.wd_sf, b.used, b.stride};
  memcpy(out, v, sizeof v);
  return FT_OK;
}

template <class T>
static ft_status dev_alloc(T** p, size_t n) {
  *p = nullptr;
  if (n == 0) return FT_OK;
  CUDA_TRY(cudaMalloc((void**)p, n * sizeof(T)));
  return FT_OK;
}

#define FT_TRY(expr)            \
  do {                          \
    ft_status s_ = (expr);      \
    if (s_ != FT_OK) return s_; \
  } while (0)

// physical memory under the arena so that `slots` slots are backed
static ft_status arena_map(ft_ctx* c, int64_t slots) {
  size_t need = (size_t)slots * (size_t)c->stride;
  size_t nchunks = (need + c->chunk - 1) / c->chunk;
  if (nchunks * c->chunk > c->va_size) return fail(FT_ERR_NO_SPACE, "cache budget exceeds the reserved arena");
  while (c->chunks.size() > nchunks) {
    size_t i = c->chunks.size() - 1;
    CU_TRY(c->drv.memUnmap(c->va + i * c->chunk, c->chunk));
    CU_TRY(c->drv.memRelease(c->chunks[i]));
    c->chunks.pop_back();
  }
  while (c->chunks.size() < nchunks) {
    size_t i = c->chunks.size();
    CUmemAllocationProp prop{};
    prop.type = CU_MEM_ALLOCATION_TYPE_PINNED;
    prop.location.type = CU_MEM_LOCATION_TYPE_DEVICE;
    prop.location.id = c->device;
    CUmemGenericAllocationHandle h;
    CUresult r = c->drv.memCreate(&h, c->chunk, &prop, 0);
    if (r != CUDA_SUCCESS) return fail(FT_ERR_CUDA, "cuMemCreate of %zu bytes failed (%d)", c->chunk, (int)r);
    r = c->drv.memMap(c->va + i * c->chunk, c->chunk, 0, h, 0);
    if (r != CUDA_SUCCESS) {
      c->drv.memRelease(h);
      return fail(FT_ERR_CUDA, "cuMemMap failed (%d)", (int)r);
    }
    CUmemAccessDesc acc{};
    acc.location.type = CU_MEM_LOCATION_TYPE_DEVICE;
    acc.location.id = c->device;
    acc.flags = CU_MEM_ACCESS_FLAGS_PROT_READWRITE;
    r = c->drv.memSetAccess(c->va + i * c->chunk, c->chunk, &acc, 1);
    if (r != CUDA_SUCCESS) {  // undo this chunk's mapping; the chunks before it stay recorded
      c->drv.memUnmap(c->va + i * c->chunk, c->chunk);
      c->drv.memRelease(h);
      return fail(FT_ERR_CUDA, "cuMemSetAccess failed (%d)", (int)r);
    }
    c->chunks.push_back(h);
  }
  c->stats.mapped_bytes = (int64_t)(c->chunks.size() * c->chunk);
  return FT_OK;
}

static uint8_t* slot_ptr(ft_ctx* c, int32_t slot) { return (uint8_t*)(c->va + (size_t)slot * (size_t)c->stride); }

extern "C" ft_status ft_create(const ft_model_desc* desc, const void* const* host_layers,
                               const void* const* resident_layers, ft_ctx** out) {
  FT_TRY(check_desc(desc));
  if (!out) return fail(FT_ERR_INVALID, "out is NULL");
  *out = nullptr;
  if (resident_layers)
    for (int l = 0; l < desc->n_layers; l++)
      if (!aligned16(resident_layers[l]))
        return fail(FT_ERR_INVALID, "resident pool of layer %d must start on a 16-byte boundary", l);
  ft_ctx* c = new ft_ctx();
  c->d = *desc;
  const int H = desc->hidden, I = desc->inter, E = desc->n_experts, k = desc->top_k, L = desc->n_layers;
  c->lay = blob_layout(H, I, desc->weight_format);
  c->stride = c->lay.stride;
  c->n_blobs = E + desc->n_shared;
  c->max_tokens = desc->max_tokens;
  c->decode_max_t = std::min(desc->max_tokens, kDecodeMaxTokens);
  auto bail = [&](ft_status st) {
    std::string keep = g_err;
    ft_destroy(c);
    g_err = keep;
    return st;
  };
  if (cudaGetDevice(&c->device) != cudaSuccess) return bail(fail(FT_ERR_CUDA, "no CUDA device"));
  if (cudaStreamCreateWithFlags(&c->copy_stream, cudaStreamNonBlocking) != cudaSuccess)
    return bail(fail(FT_ERR_CUDA, "copy stream"));

  c->host_layers.assign(L, nullptr);
  c->resident.assign(L, nullptr);
  for (int l = 0; l < L; l++) {
    if (host_layers) c->host_layers[l] = (const uint8_t*)host_layers[l];
    if (resident_layers) c->resident[l] = (const uint8_t*)resident_layers[l];
  }
  // pin pageable host pools
  for (int l = 0; l < L; l++) {
    const uint8_t* hp = c->host_layers[l];
    if (!hp) continue;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, hp) == cudaSuccess && at.type == cudaMemoryTypeHost) continue;
    cudaGetLastError();
    if (cudaHostRegister((void*)hp, (size_t)c->n_blobs * c->stride, cudaHostRegisterDefault) != cudaSuccess)
      return bail(fail(FT_ERR_CUDA, "cudaHostRegister of layer %d pool failed", l));
    c->registered.push_back((void*)hp);
  }

  const int T = desc->max_tokens;
  ft_status st;
  if ((st = dev_alloc(&c->d_status, 1)) || (st = dev_alloc(&c->d_flag, 1)) || (st = dev_alloc(&c->d_qamax, 1)) ||
      (st = dev_alloc(&c->d_logits, (size_t)T * E)) ||
      (st = dev_alloc(&c->d_ids, (size_t)T * k)) || (st = dev_alloc(&c->d_w, (size_t)T * k)) ||
      (st = dev_alloc(&c->d_offs, E + 1)) || (st = dev_alloc(&c->d_perm, (size_t)T * k)) ||
      (st = dev_alloc(&c->d_inv, (size_t)T * k)) || (st = dev_alloc(&c->d_active, E)) ||
      (st = dev_alloc(&c->d_nact, 1)) || (st = dev_alloc(&c->d_pad_offs, E + 2)) ||
      (st = dev_alloc(&c->d_h, (size_t)(c->decode_max_t * k + desc->n_shared * c->decode_max_t) * I)) ||
      (st = dev_alloc(&c->d_y, (size_t)(c->decode_max_t * k + desc->n_shared * c->decode_max_t) * H)) ||
      (st = dev_alloc(&c->d_counters, (size_t)H / 8)) ||
      (st = dev_alloc(&c->d_routes, (size_t)L)) ||
      (st = dev_alloc(&c->d_xbuf[0], (size_t)c->decode_max_t * H)) ||
      (st = dev_alloc(&c->d_xbuf[1], (size_t)c->decode_max_t * H)))
    return bail(st);
  if (stack_supported(H, I, 1)) {
    c->sync_stride = stack_sync_stride(H, I);
    const int t2 = std::min(c->decode_max_t, 2);
    const size_t hrows = (size_t)(t2 * k + desc->n_shared * t2);
    c->tagged_words = (int64_t)(hrows * I + (size_t)t2 * H / 2);
    if ((st = dev_alloc(&c->d_sync, (size_t)L * c->sync_stride)) ||
        (st = dev_alloc(&c->d_tagged, (size_t)c->tagged_words)) || (st = dev_alloc(&c->d_epoch, 1)))
      return bail(st);
    c->d_h_tagged = c->d_tagged;
    c->d_x_tagged = c->d_tagged + hrows * I;
    if (cudaMemset(c->d_tagged, 0, (size_t)c->tagged_words * sizeof(uint64_t)) != cudaSuccess ||
        cudaMemset(c->d_epoch, 0, sizeof(uint32_t)) != cudaSuccess)
      return bail(fail(FT_ERR_CUDA, "memset"));
  }
  if (cudaMemset(c->d_counters, 0, (size_t)H / 8 * sizeof(int)) != cudaSuccess)
    return bail(fail(FT_ERR_CUDA, "memset"));
  if (cudaMemset(c->d_status, 0, sizeof(int)) != cudaSuccess || cudaMemset(c->d_flag, 0, sizeof(int)) != cudaSuccess)
    return bail(fail(FT_ERR_CUDA, "memset"));
  if (cudaMallocHost(&c->h_ids, (size_t)T * k * sizeof(int32_t)) != cudaSuccess ||
      cudaMallocHost(&c->h_status, sizeof(int)) != cudaSuccess)
    return bail(fail(FT_ERR_CUDA, "pinned scratch"));
  if (cudaEventCreateWithFlags(&c->ev_ids, cudaEventDisableTiming) != cudaSuccess)
    return bail(fail(FT_ERR_CUDA, "event"));
  for (int b = 0; b < 2; b++) {
    if (cudaEventCreateWithFlags(&c->ev_landed[b], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c->ev_done[b], cudaEventDisableTiming) != cudaSuccess)
      return bail(fail(FT_ERR_CUDA, "event"));
  }

  // resident pointer table
  bool any_resident = false, any_host_only = false;
  std::vector<const uint8_t*> tab((size_t)L * c->n_blobs, nullptr);
  for (int l = 0; l < L; l++) {
    if (c->resident[l]) {
      any_resident = true;
      for (int e = 0; e < c->n_blobs; e++) tab[(size_t)l * c->n_blobs + e] = c->resident[l] + (size_t)e * c->stride;
    } else if (c->host_layers[l]) {
      any_host_only = true;
    }
  }
  if (any_resident) {
    if ((st = dev_alloc(&c->d_eptr_res, tab.size()))) return bail(st);
    if (cudaMemcpy(c->d_eptr_res, tab.data(), tab.size() * sizeof(void*), cudaMemcpyHostToDevice) != cudaSuccess)
      return bail(fail(FT_ERR_CUDA, "resident table"));
  }

  // expert cache over a reserved virtual range
  if (desc->cache_budget_bytes > 0 && any_host_only) {
    if ((st = load_driver(c->drv))) return bail(st);
    CUmemAllocationProp prop{};
    prop.type = CU_MEM_ALLOCATION_TYPE_PINNED;
    prop.location.type = CU_MEM_LOCATION_TYPE_DEVICE;
    prop.location.id = c->device;
    size_t gran = 0;
    if (c->drv.memGetAllocationGranularity(&gran, &prop, CU_MEM_ALLOC_GRANULARITY_RECOMMENDED) != CUDA_SUCCESS)
      return bail(fail(FT_ERR_CUDA, "granularity"));
    c->chunk = pad_up(kArenaChunkBytes, gran);
    size_t total = 0, freeb = 0;
    cudaMemGetInfo(&freeb, &total);
    size_t pool = (size_t)L * c->n_blobs * c->stride;
    c->va_size = pad_up(std::min(pool, total) + c->chunk, c->chunk);
    if (c->drv.memAddressReserve(&c->va, c->va_size, c->chunk, 0, 0) != CUDA_SUCCESS)
      return bail(fail(FT_ERR_CUDA, "cuMemAddressReserve of %zu bytes failed", c->va_size));
    c->cache_on = true;
    c->sel_count.assign((size_t)L * E, 0);
    int64_t cap = desc->cache_budget_bytes / c->stride;
    c->lru.set_capacity(cap);
    if ((st = arena_map(c, cap))) return bail(st);
    c->stats.capacity_slots = cap;
    if (cudaMallocHost(&c->h_eptr_cache, (size_t)L * c->n_blobs * sizeof(void*)) != cudaSuccess)
      return bail(fail(FT_ERR_CUDA, "pinned table"));
    memset(c->h_eptr_cache, 0, (size_t)L * c->n_blobs * sizeof(void*));
    if ((st = dev_alloc(&c->d_eptr_cache, (size_t)L * c->n_blobs))) return bail(st);
    // shared experts stay resident outside the LRU
    if (desc->n_shared > 0) {
      if ((st = dev_alloc(&c->d_shared, (size_t)L * desc->n_shared * c->stride))) return bail(st);
      for (int l = 0; l < L; l++) {
        if (!c->host_layers[l]) continue;
        for (int s = 0; s < desc->n_shared; s++) {
          uint8_t* dst = c->d_shared + ((size_t)l * desc->n_shared + s) * c->stride;
          if (cudaMemcpy(dst, c->host_layers[l] + (size_t)(E + s) * c->stride, c->stride, cudaMemcpyHostToDevice) !=
              cudaSuccess)
            return bail(fail(FT_ERR_CUDA, "shared expert copy"));
          c->h_eptr_cache[(size_t)l * c->n_blobs + E + s] = dst;
        }
      }
    }
    if (cudaMemcpy(c->d_eptr_cache, c->h_eptr_cache, (size_t)L * c->n_blobs * sizeof(void*), cudaMemcpyHostToDevice) !=
        cudaSuccess)
      return bail(fail(FT_ERR_CUDA, "cache table"));
  }
  for (int b = 0; b < 2; b++) cudaEventRecord(c->ev_done[b], c->copy_stream);
  if (cudaDeviceSynchronize() != cudaSuccess) return bail(fail(FT_ERR_CUDA, "create sync"));
  *out = c;
  return FT_OK;
}

extern "C" ft_status ft_destroy(ft_ctx* c) {
  if (!c) return FT_OK;
  cudaDeviceSynchronize();
  for (auto* v : {&c->tmarks, &c->gmarks})
    for (auto& m : *v) {
      cudaEventDestroy(m.second.first);
      cudaEventDestroy(m.second.second);
    }
  for (auto& st : c->copy_timing)
    for (cudaEvent_t e : {st.ref, st.c0, st.c1, st.h0, st.h1})
      if (e) cudaEventDestroy(e);
  for (cudaEvent_t e : c->spare_events) cudaEventDestroy(e);
  for (cudaEvent_t e : c->miss_events) cudaEventDestroy(e);
  for (cudaEvent_t e : c->spare_miss_events) cudaEventDestroy(e);
  for (auto& kv : c->pending) cudaEventDestroy(kv.second);
  free_prefill_scratch(c->pf);
  cudaFree(c->d_status);
  cudaFree(c->d_flag);
  cudaFree(c->d_qamax);
  cudaFree(c->d_logits);
  cudaFree(c->d_ids);
  cudaFree(c->d_w);
  cudaFree(c->d_offs);
  cudaFree(c->d_perm);
  cudaFree(c->d_inv);
  cudaFree(c->d_active);
  cudaFree(c->d_nact);
  cudaFree(c->d_pad_offs);
  cudaFree(c->d_h);
  cudaFree(c->d_y);
  cudaFree(c->d_counters);
  cudaFree(c->d_routes);
  cudaFree(c->d_xbuf[0]);
  cudaFree(c->d_xbuf[1]);
  cudaFree(c->d_sync);
  cudaFree(c->d_tagged);
  cudaFree(c->d_epoch);
  cudaFree(c->d_eptr_res);
  cudaFree(c->d_eptr_cache);
  cudaFree(c->d_shared);
  for (int b = 0; b < 2; b++) {
    cudaFree(c->d_stage[b]);
    cudaFree(c->d_eptr_stage[b]);
    if (c->ev_landed[b]) cudaEventDestroy(c->ev_landed[b]);
    if (c->ev_done[b]) cudaEventDestroy(c->ev_done[b]);
  }
  if (c->h_eptr_cache) cudaFreeHost(c->h_eptr_cache);
  if (c->h_ids) cudaFreeHost(c->h_ids);
  if (c->h_status) cudaFreeHost(c->h_status);
  if (c->ev_ids) cudaEventDestroy(c->ev_ids);
  if (c->va) {
    for (size_t i = 0; i < c->chunks.size(); i++) {
      c->drv.memUnmap(c->va + i * c->chunk, c->chunk);
      c->drv.memRelease(c->chunks[i]);
    }
    c->drv.memAddressFree(c->va, c->va_size);
  }
  for (void* p : c->registered) cudaHostUnregister(p);
  if (c->copy_stream) cudaStreamDestroy(c->copy_stream);
  delete c;
  cudaGetLastError();
  return FT_OK;
}

// bounded host wait on an event: polls, gives up after `limit` seconds
// Bounded host wait on an event: polls without sleeping for the first
// kHostSpinSeconds (a decode layer's wait for its routed ids is tens of
// microseconds, and a short sleep lasts tens of microseconds more than asked
// on a stock kernel timer), then sleeps between polls until `limit`.
static ft_status wait_event(cudaEvent_t ev, const char* what, double limit) {
  const auto t0 = std::chrono::steady_clock::now();
  while (true) {
    cudaError_t q = cudaEventQuery(ev);
    if (q == cudaSuccess) return FT_OK;
    if (q != cudaErrorNotReady) return fail(FT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(q));
    const double s = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
    if (s > limit) return fail(FT_ERR_TIMEOUT, "%s: gave up after %.3f s", what, s);
    if (s > kHostSpinSeconds) std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
}

static ft_status status_to_ft(int st) {
  if (st & kStNonfinite) return fail(FT_ERR_NONFINITE, "NaN or +inf router logit (or no finite logit in a row)");
  if (st & kStBadId) return fail(FT_ERR_INVALID, "expert id out of range");
  if (st & kStMissing) return fail(FT_ERR_NOT_FOUND, "an expert blob pointer was NULL at kernel time");
  if (st & kStTimeout) return fail(FT_ERR_TIMEOUT, "a device wait gave up");
  return FT_OK;
}

extern "C" ft_status ft_sync_status(ft_ctx* c, void* stream) {
  if (!c) return fail(FT_ERR_INVALID, "ctx is NULL");
  cudaStream_t s = (cudaStream_t)stream;
  CUDA_TRY(cudaMemcpyAsync(c->h_status, c->d_status, sizeof(int), cudaMemcpyDeviceToHost, s));
  CUDA_TRY(cudaMemsetAsync(c->d_status, 0, sizeof(int), s));
  CUDA_TRY(cudaStreamSynchronize(s));
  return status_to_ft(*c->h_status);
}

// ---------------------------------------------------------------------------
// single steps
// ---------------------------------------------------------------------------
extern "C" ft_status ft_router_logits(ft_ctx* c, const void* x, int64_t T, int32_t H, const float* wr, int32_t E,
                                      float* logits, void* stream) {
  if (!c || (!x && T > 0) || !wr || !logits) return fail(FT_ERR_INVALID, "NULL argument");
  if (T < 0 || H <= 0 || H % 128 || E <= 0) return fail(FT_ERR_INVALID, "bad shape T=%lld H=%d E=%d", (long long)T, H, E);
  if (!aligned16(x) || !aligned16(wr) || !aligned16(logits))
    return fail(FT_ERR_INVALID, "x, wr and logits must start on a 16-byte boundary");
  CUDA_TRY(launch_router_logits((const uint16_t*)x, wr, (int)T, H, E, logits, (cudaStream_t)stream));
  return FT_OK;
}

extern "C" ft_status ft_moe_route(ft_ctx* c, const float* logits, int64_t T, int32_t E, int32_t k, uint32_t flags,
                                  int32_t* ids, float* w, void* stream) {
  if (!c || !logits || !ids || !w) return fail(FT_ERR_INVALID, "NULL argument");
  if (T < 0 || E <= 0 || E > 1024 || k <= 0 || k > 16 || k > E) return fail(FT_ERR_INVALID, "bad shape E=%d k=%d", E, k);
  CUDA_TRY(launch_topk(logits, (int)T, E, k, (flags & FT_ROUTE_RENORM) ? 1 : 0, ids, w, c->d_status,
                       (cudaStream_t)stream));
  return FT_OK;
}

extern "C" ft_status ft_moe_permute(ft_ctx* c, const int32_t* ids, int64_t T, int32_t k, int32_t E, int32_t* offs,
                                    int32_t* perm, int32_t* inv, void* stream) {
  if (!c || !ids || !offs || !perm || !inv) return fail(FT_ERR_INVALID, "NULL argument");
  if (T < 0 || E <= 0 || E > 1024 || k <= 0) return fail(FT_ERR_INVALID, "bad shape");
  if (E > c->d.n_experts) {
    return fail(FT_ERR_INVALID, "E=%d larger than the context's n_experts %d (scratch)", E, c->d.n_experts);
  }
  CUDA_TRY(launch_permute(ids, (int)(T * k), E, offs, perm, inv, c->d_active, c->d_nact, nullptr, c->d_status,
                          (cudaStream_t)stream));
  return FT_OK;
}

extern "C" ft_status ft_quantize_mxfp4(ft_ctx* c, const float* x, int64_t R, int32_t K, uint8_t* codes,
                                       uint8_t* scales, void* stream) {
  if (!c || (!x && R > 0) || !codes || !scales) return fail(FT_ERR_INVALID, "NULL argument");
  if (R < 0 || K <= 0 || K % 128) return fail(FT_ERR_INVALID, "K=%d not a positive multiple of 128", K);
  if (!aligned16(x) || !aligned16(codes)) return fail(FT_ERR_INVALID, "x and codes must start on a 16-byte boundary");
  CUDA_TRY(launch_quantize_rows(x, R, K, codes, scales, (cudaStream_t)stream));
  return FT_OK;
}

extern "C" ft_status ft_quantize_nvfp4(ft_ctx* c, const float* x, int64_t R, int32_t K, uint8_t* codes,
                                       uint8_t* scales, float* tensor_scale, void* stream) {
  if (!c || (!x && R > 0) || !codes || !scales || !tensor_scale) return fail(FT_ERR_INVALID, "NULL argument");
  if (R < 0 || K <= 0 || K % 128) return fail(FT_ERR_INVALID, "K=%d not a positive multiple of 128", K);
  if (!aligned16(x) || !aligned16(codes)) return fail(FT_ERR_INVALID, "x and codes must start on a 16-byte boundary");
  CUDA_TRY(launch_quantize_rows_nv(x, R, K, c->d_qamax, codes, scales, tensor_scale, (cudaStream_t)stream));
  c->last_stream = (cudaStream_t)stream;
  return FT_OK;
}

extern "C" ft_status ft_debug_dequant(ft_ctx* c, const void* blob, int32_t mat, float* out, void* stream) {
  if (!c || !blob || !out || mat < 0 || mat > 2) return fail(FT_ERR_INVALID, "bad argument");
  if (!decode_supported(c->d.hidden, c->d.inter))
    return fail(FT_ERR_INVALID, "the decode tile does not take hidden %d / inter %d", c->d.hidden, c->d.inter);
  CUDA_TRY(launch_dec_dequant((const uint8_t*)blob, c->lay, mat, c->d.hidden, c->d.inter, out, (cudaStream_t)stream));
  return FT_OK;
}

extern "C" ft_status ft_decode_geometry(int32_t hidden, int32_t inter, int32_t n_layers, int64_t out[24]) {
  if (!out) return fail(FT_ERR_INVALID, "out is NULL");
  if (hidden <= 0 || inter <= 0 || hidden % 128 || inter % 128 || n_layers <= 0)
    return fail(FT_ERR_INVALID, "hidden %d / inter %d not positive multiples of 128, or n_layers %d", hidden, inter,
                n_layers);
  decode_geometry(hidden, inter, out);
  out[22] = stack_supported(hidden, inter, n_layers) ? 1 : 0;
  out[23] = out[22] ? stack_sync_stride(hidden, inter) : 0;
  return FT_OK;
}

namespace ft {
size_t fp4_probe_smem();
cudaError_t launch_fp4_probe(int64_t iters, float* sink, int* status, int* grid_out, cudaStream_t s);
}  // namespace ft

extern "C" ft_status ft_fp4_mma_probe(int64_t iters, float* sink, int32_t* status, int32_t* grid, void* stream) {
  if (!sink || !status || !grid) return fail(FT_ERR_INVALID, "NULL argument");
  if (iters < 1 || iters > 65536) return fail(FT_ERR_INVALID, "iters %lld outside [1, 65536]", (long long)iters);
  int g = 0;
  CUDA_TRY(launch_fp4_probe(iters, sink, status, &g, (cudaStream_t)stream));
  *grid = g;
  return FT_OK;
}

extern "C" ft_status ft_flow_geometry(int32_t hidden, int32_t inter, int32_t T, int32_t top_k, int32_t n_shared,
                                      int32_t n_experts, int32_t n_layers, int32_t weight_format, int64_t out[3]) {
  if (!out) return fail(FT_ERR_INVALID, "out is NULL");
  if (hidden <= 0 || inter <= 0 || hidden % 128 || inter % 128 || top_k <= 0 || top_k > 16 || n_experts <= 0 ||
      n_shared < 0 || n_shared > 1 || T <= 0 || n_layers <= 0 || weight_format < 0 || weight_format > 2)
    return fail(FT_ERR_INVALID, "bad shape");
  const FlowGeom fg = flow_geometry(hidden, inter, T, top_k, n_shared, n_experts, n_layers, weight_format);
  out[0] = fg.ok ? 1 : 0;
  out[1] = fg.rows_cap;
  out[2] = (int64_t)fg.smem;
  return FT_OK;
}

extern "C" ft_status ft_debug_device_wait(ft_ctx* c, int64_t timeout_us, void* stream) {
  if (!c) return fail(FT_ERR_INVALID, "ctx is NULL");
  if (timeout_us < 1 || timeout_us > 2000000) return fail(FT_ERR_INVALID, "timeout_us %lld outside [1, 2e6]", (long long)timeout_us);
  CUDA_TRY(launch_debug_wait(c->d_flag, c->d_status, (uint64_t)timeout_us * 1000u, (cudaStream_t)stream));
  c->last_stream = (cudaStream_t)stream;
  return FT_OK;
}

extern "C" ft_status ft_debug_stack_epoch(ft_ctx* c, uint32_t epoch, int32_t poison_layer) {
  if (!c) return fail(FT_ERR_INVALID, "ctx is NULL");
  if (!c->d_epoch) return fail(FT_ERR_STATE, "this context has no persistent decode kernel");
  if (poison_layer > 127) return fail(FT_ERR_INVALID, "poison_layer %d above 127", poison_layer);
  CUDA_TRY(cudaDeviceSynchronize());
  CUDA_TRY(cudaMemcpy(c->d_epoch, &epoch, sizeof(epoch), cudaMemcpyHostToDevice));
  if (poison_layer >= 0) {
    const uint32_t tag = (next_epoch(epoch, nullptr) << 7) | (uint32_t)poison_layer;
    const uint64_t word = ((uint64_t)tag << 32) | 0x7fc00000ull;  // a NaN under the next launch's tag
    std::vector<uint64_t> w((size_t)c->tagged_words, word);
    CUDA_TRY(cudaMemcpy(c->d_tagged, w.data(), w.size() * sizeof(uint64_t), cudaMemcpyHostToDevice));
  }
  return FT_OK;
}

extern "C" ft_status ft_debug_stack_timeline(ft_ctx* c, uint64_t* buf, int64_t n_words) {
  if (!c) return fail(FT_ERR_INVALID, "ctx is NULL");
  if (buf && n_words <= 0) return fail(FT_ERR_INVALID, "n_words must be positive");
  c->timeline = buf;
  c->timeline_words = buf ? n_words : 0;
  return FT_OK;
}

extern "C" ft_status ft_debug_host_wait_limit(ft_ctx* c, double seconds) {
  if (!c) return fail(FT_ERR_INVALID, "ctx is NULL");
  if (!(seconds > 0.0)) return fail(FT_ERR_INVALID, "limit must be positive");
  c->host_wait_s = seconds;
  return FT_OK;
}

extern "C" ft_status ft_debug_fail_copy(ft_ctx* c, int64_t n) {
  if (!c) return fail(FT_ERR_INVALID, "ctx is NULL");
  if (n < 0) return fail(FT_ERR_INVALID, "n must be >= 0");
  c->fail_copy_in = n;
  return FT_OK;
}

// ---------------------------------------------------------------------------
// expert cache
// ---------------------------------------------------------------------------
// Between two reads the trace keeps at most kTraceMaxEvents events; later
// ones are counted and dropped, so a run that never reads it stays bounded.
static void record(ft_ctx* c, int kind, int layer, int expert, int slot, int from) {
  if ((int64_t)c->trace.size() >= kTraceMaxEvents) {
    c->trace_dropped++;
    return;
  }
  c->trace.push_back(ft_cache_event{kind, layer, expert, slot, from});
}

static int64_t key_of(ft_ctx* c, int layer, int expert) { return (int64_t)layer * c->d.n_experts + expert; }

// Evict the least recent key not in `keep` (may be empty); returns its slot
// (-1 if none) and the evicted key in *victim.
static int32_t evict_one(ft_ctx* c, const std::vector<int64_t>& keep, int64_t* victim = nullptr,
                         int skip_layer = -1) {
  for (auto it = c->lru.order.begin(); it != c->lru.order.end(); ++it) {
    int64_t key = *it;
    if (std::find(keep.begin(), keep.end(), key) != keep.end()) continue;
    if (skip_layer >= 0 && key / c->d.n_experts == skip_layer) continue;
    auto m = c->lru.map.find(key);
    c->unused_prefetch.erase(key);
    auto pe = c->pending.find(key);
    if (pe != c->pending.end()) {  // a later copy into the slot is ordered after it on the copy stream
      c->spare_miss_events.push_back(pe->second);
      c->pending.erase(pe);
    }
    int32_t slot = m->second.first;
    c->lru.order.erase(it);
    c->lru.map.erase(m);
    c->lru.slot_used[slot] = 0;
    int layer = (int)(key / c->d.n_experts), e = (int)(key % c->d.n_experts);
    c->h_eptr_cache[(size_t)layer * c->n_blobs + e] = nullptr;
    record(c, FT_EV_EVICT, layer, e, slot, -1);
    c->stats.evictions++;
    if (victim) *victim = key;
    return slot;
  }
  return -1;
}

// Timing of the miss copies: each cache step with a miss records a (start,
// end) event pair around its copies on the copy stream.  Pairs finish in
// issue order; finished ones are folded into stats.h2d_ms and their events
// reused, so a long run holds only the pairs still in flight.
static void fold_copy_timing(ft_ctx* c) {
  size_t n = 0;
  for (; n < c->copy_timing.size(); n++) {
    const auto& st = c->copy_timing[n];
    if (cudaEventQuery(st.c1) != cudaSuccess || (st.h1 && cudaEventQuery(st.h1) != cudaSuccess)) break;
    float c0 = 0.f, c1 = 0.f;
    if (cudaEventElapsedTime(&c0, st.ref, st.c0) == cudaSuccess && cudaEventElapsedTime(&c1, st.ref, st.c1) == cudaSuccess) {
      c->stats.h2d_ms += c1 - c0;
      float h0 = 0.f, h1 = 0.f;
      if (st.h0 && cudaEventElapsedTime(&h0, st.ref, st.h0) == cudaSuccess &&
          cudaEventElapsedTime(&h1, st.ref, st.h1) == cudaSuccess) {
        c->stats.hit_ms += h1 - h0;
        c->stats.overlap_ms += std::max(0.f, std::min(c1, h1) - std::max(c0, h0));
      }
    }
    for (cudaEvent_t e : {st.ref, st.c0, st.c1, st.h0, st.h1})
      if (e) c->spare_events.push_back(e);
  }
  c->copy_timing.erase(c->copy_timing.begin(), c->copy_timing.begin() + (std::ptrdiff_t)n);
}

static cudaEvent_t copy_event(ft_ctx* c) {
  if (!c->spare_events.empty()) {
    cudaEvent_t e = c->spare_events.back();
    c->spare_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// An event (no timing) marking the end of one miss's copy on the copy stream.
static cudaEvent_t miss_event(ft_ctx* c) {
  cudaEvent_t e = nullptr;
  if (!c->spare_miss_events.empty()) {
    e = c->spare_miss_events.back();
    c->spare_miss_events.pop_back();
  } else {
    cudaEventCreateWithFlags(&e, cudaEventDisableTiming);
  }
  c->miss_events.push_back(e);
  return e;
}

// Issue the H2D copy of (layer, e) into `slot` on the copy stream.
static ft_status fetch(ft_ctx* c, int layer, int e, int32_t slot) {
  if (c->fail_copy_in > 0 && --c->fail_copy_in == 0)
    return fail(FT_ERR_CUDA, "injected failure of the host-to-device copy of expert (%d, %d)", layer, e);
  const uint8_t* src = c->host_layers[layer] + (size_t)e * c->stride;
  CUDA_TRY(cudaMemcpyAsync(slot_ptr(c, slot), src, (size_t)c->lay.used, cudaMemcpyHostToDevice, c->copy_stream));
  c->stats.h2d_bytes += c->lay.used;
  return FT_OK;
}

// One decode step of the cache for `layer` over the distinct experts S (ascending).
// Misses are fetched in ascending expert id; for each, miss_units gets its
// position in S and c->miss_events an event after its copy.  `ref` (a timing
// event that precedes the step, or NULL) anchors the step's timing.
static ft_status cache_step(ft_ctx* c, int layer, const std::vector<int>& S, bool& any_miss, std::vector<int>& dirty,
                            std::vector<int>* miss_units = nullptr, cudaEvent_t ref = nullptr) {
  any_miss = false;
  if ((int64_t)S.size() > c->lru.capacity)
    return fail(FT_ERR_NO_SPACE, "%zu experts in one step exceed the cache capacity of %lld slots", S.size(),
                (long long)c->lru.capacity);
  fold_copy_timing(c);
  std::vector<int64_t> keep;
  keep.reserve(S.size());
  for (int e : S) keep.push_back(key_of(c, layer, e));
  cudaEvent_t t0 = nullptr, t1 = nullptr;
  for (size_t si = 0; si < S.size(); si++) {
    const int e = S[si];
    int64_t key = key_of(c, layer, e);
    auto m = c->lru.map.find(key);
    if (m != c->lru.map.end()) {
      c->lru.order.splice(c->lru.order.end(), c->lru.order, m->second.second);
      record(c, FT_EV_HIT, layer, e, m->second.first, -1);
      c->stats.hits++;
      if (c->unused_prefetch.erase(key)) c->stats.prefetch_hits++;
      auto pe = c->pending.find(key);
      if (pe != c->pending.end()) {
        if (cudaEventQuery(pe->second) == cudaSuccess) {
          c->spare_miss_events.push_back(pe->second);
        } else if (miss_units) {  // its prefetch copy is still in flight: the expert waits for it
          miss_units->push_back((int)si);
          c->miss_events.push_back(pe->second);
        } else {
          cudaEventSynchronize(pe->second);
          c->spare_miss_events.push_back(pe->second);
        }
        c->pending.erase(pe);
      }
      continue;
    }
    int32_t slot;
    if ((int64_t)c->lru.map.size() >= c->lru.capacity) {
      int64_t victim = -1;
      slot = evict_one(c, keep, &victim);
      if (slot < 0) return fail(FT_ERR_NO_SPACE, "no evictable key");
      dirty.push_back((int)(victim / c->d.n_experts));
    } else {
      slot = c->lru.lowest_free();
    }
    if (!any_miss) {
      if (!ref) {  // a step without a caller's anchor is anchored at its first copy
        ref = copy_event(c);
        cudaEventRecord(ref, c->copy_stream);
      }
      t0 = copy_event(c);
      t1 = copy_event(c);
      cudaEventRecord(t0, c->copy_stream);
    }
    any_miss = true;
    c->lru.order.push_back(key);
    c->lru.map[key] = {slot, std::prev(c->lru.order.end())};
    c->lru.slot_used[slot] = 1;
    c->h_eptr_cache[(size_t)layer * c->n_blobs + e] = slot_ptr(c, slot);
    record(c, FT_EV_MISS, layer, e, slot, -1);
    c->stats.misses++;
    const ft_status fs = fetch(c, layer, e, slot);
    if (fs != FT_OK) {
      // the key never became resident: drop it again; keys fetched earlier
      // in this step stay (their copies are queued on the copy stream)
      c->lru.order.pop_back();
      c->lru.map.erase(key);
      c->lru.slot_used[slot] = 0;
      c->h_eptr_cache[(size_t)layer * c->n_blobs + e] = nullptr;
      record(c, FT_EV_EVICT, layer, e, slot, -1);
      c->stats.evictions++;
      c->stats.used_slots = (int64_t)c->lru.map.size();
      cudaEventRecord(t1, c->copy_stream);
      c->copy_timing.push_back({ref, t0, t1, nullptr, nullptr});
      // a later step counts the earlier keys as hits and does not wait for
      // their copies: let them land now
      cudaStreamSynchronize(c->copy_stream);
      return fs;
    }
    if (miss_units) {
      miss_units->push_back((int)si);
      cudaEventRecord(miss_event(c), c->copy_stream);
    }
  }
  if (any_miss) {
    cudaEventRecord(t1, c->copy_stream);
    c->copy_timing.push_back({ref, t0, t1, nullptr, nullptr});
  } else if (ref) {
    c->spare_events.push_back(ref);
  }
  c->stats.used_slots = (int64_t)c->lru.map.size();
  return FT_OK;
}

static ft_status push_table_rows(ft_ctx* c, const std::vector<int>& rows, cudaStream_t s) {
  std::vector<int> r = rows;
  std::sort(r.begin(), r.end());
  r.erase(std::unique(r.begin(), r.end()), r.end());
  for (int l : r)
    CUDA_TRY(cudaMemcpyAsync(c->d_eptr_cache + (size_t)l * c->n_blobs, c->h_eptr_cache + (size_t)l * c->n_blobs,
                             c->n_blobs * sizeof(void*), cudaMemcpyHostToDevice, s));
  return FT_OK;
}

// Decode-time next-layer prefetch (see ft_cache_prefetch in ft_moe.h).
static ft_status prefetch_next(ft_ctx* c, int layer, const std::vector<int>& S) {
  const int E = c->d.n_experts, L = c->d.n_layers;
  for (int e : S) c->sel_count[(size_t)layer * E + e]++;
  if (c->prefetch_per_layer <= 0) return FT_OK;
  const int n = (layer + 1) % L;
  if (!c->host_layers[n] || c->resident[n]) return FT_OK;
  std::vector<int> cand;
  for (int e = 0; e < E; e++)
    if (c->sel_count[(size_t)n * E + e] > 0) cand.push_back(e);
  const int64_t* cnt = c->sel_count.data() + (size_t)n * E;
  std::stable_sort(cand.begin(), cand.end(), [&](int a, int b) { return cnt[a] > cnt[b]; });
  std::vector<int64_t> keep;
  for (int e : S) keep.push_back(key_of(c, layer, e));
  int done = 0;
  for (int e : cand) {
    if (done >= c->prefetch_per_layer) break;
    const int64_t key = key_of(c, n, e);
    if (c->lru.map.count(key)) continue;
    if (c->lru.capacity <= 0) break;
    int32_t slot;
    if ((int64_t)c->lru.map.size() >= c->lru.capacity) {
      slot = evict_one(c, keep, nullptr, n);
      if (slot < 0) break;
    } else {
      slot = c->lru.lowest_free();
    }
    c->lru.order.push_back(key);
    c->lru.map[key] = {slot, std::prev(c->lru.order.end())};
    c->lru.slot_used[slot] = 1;
    c->h_eptr_cache[(size_t)n * c->n_blobs + e] = slot_ptr(c, slot);
    record(c, FT_EV_PREFETCH, n, e, slot, -1);
    const ft_status fs = fetch(c, n, e, slot);
    c->stats.h2d_bytes -= fs == FT_OK ? c->lay.used : 0;  // demand-miss bytes only; counted below
    if (fs != FT_OK) {  // the key never became resident
      c->lru.order.pop_back();
      c->lru.map.erase(key);
      c->lru.slot_used[slot] = 0;
      c->h_eptr_cache[(size_t)n * c->n_blobs + e] = nullptr;
      record(c, FT_EV_EVICT, n, e, slot, -1);
      c->stats.evictions++;
      cudaStreamSynchronize(c->copy_stream);
      return fs;
    }
    cudaEvent_t ev = nullptr;
    if (!c->spare_miss_events.empty()) {
      ev = c->spare_miss_events.back();
      c->spare_miss_events.pop_back();
    } else {
      CUDA_TRY(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
    }
    CUDA_TRY(cudaEventRecord(ev, c->copy_stream));
    c->pending[key] = ev;
    c->unused_prefetch.insert(key);
    c->stats.prefetches++;
    c->stats.prefetch_bytes += c->lay.used;
    done++;
  }
  c->stats.used_slots = (int64_t)c->lru.map.size();
  return FT_OK;
}

extern "C" ft_status ft_cache_prefetch(ft_ctx* c, int32_t per_layer) {
  if (!c) return fail(FT_ERR_INVALID, "ctx is NULL");
  if (!c->cache_on) return fail(FT_ERR_INVALID, "context has no expert cache");
  if (per_layer < 0 || per_layer > 16) return fail(FT_ERR_INVALID, "per_layer %d outside [0, 16]", per_layer);
  c->prefetch_per_layer = per_layer;
  return FT_OK;
}

extern "C" ft_status ft_expert_cache_lookup(ft_ctx* c, int32_t layer, int32_t expert, int32_t* slot) {
  if (!c || !slot) return fail(FT_ERR_INVALID, "NULL argument");
  if (!c->cache_on) return fail(FT_ERR_INVALID, "context has no expert cache");
  if (layer < 0 || layer >= c->d.n_layers || expert < 0 || expert >= c->d.n_experts)
    return fail(FT_ERR_INVALID, "bad key (%d, %d)", layer, expert);
  auto m = c->lru.map.find(key_of(c, layer, expert));
  if (m == c->lru.map.end()) {
    *slot = -1;
    return FT_OK;
  }
  c->lru.order.splice(c->lru.order.end(), c->lru.order, m->second.second);
  *slot = m->second.first;
  record(c, FT_EV_HIT, layer, expert, *slot, -1);
  c->stats.hits++;
  return FT_OK;
}

extern "C" ft_status ft_expert_cache_insert(ft_ctx* c, int32_t layer, int32_t expert, int32_t* slot,
                                            int64_t* evicted_key, void* stream) {
  NvtxRange nvtx_range("ft_expert_cache_insert");
  if (!c || !slot) return fail(FT_ERR_INVALID, "NULL argument");
  if (!c->cache_on) return fail(FT_ERR_INVALID, "context has no expert cache");
  if (layer < 0 || layer >= c->d.n_layers || expert < 0 || expert >= c->d.n_experts)
    return fail(FT_ERR_INVALID, "bad key (%d, %d)", layer, expert);
  if (!c->host_layers[layer]) return fail(FT_ERR_NOT_FOUND, "layer %d has no host pool", layer);
  if (evicted_key) *evicted_key = -1;
  if (c->lru.capacity <= 0) return fail(FT_ERR_NO_SPACE, "cache capacity is 0");
  cudaStream_t s = (cudaStream_t)stream;
  // table rows may still be read by queued work: order after it
  if (c->last_stream) CUDA_TRY(cudaStreamSynchronize(c->last_stream));
  CUDA_TRY(cudaStreamSynchronize(s));
  std::vector<int> S{expert};
  std::vector<int> dirty{layer};
  int64_t before_evict = c->stats.evictions;
  int64_t victim = -1;
  if (c->lru.map.find(key_of(c, layer, expert)) == c->lru.map.end() && (int64_t)c->lru.map.size() >= c->lru.capacity)
    victim = c->lru.order.front();
  bool any_miss;
  FT_TRY(cache_step(c, layer, S, any_miss, dirty));
  if (evicted_key && c->stats.evictions > before_evict) *evicted_key = victim;
  *slot = c->lru.map[key_of(c, layer, expert)].first;
  if (any_miss) {
    cudaEvent_t done = c->copy_timing.back().c1;
    CUDA_TRY(cudaStreamWaitEvent(s, done, 0));
  }
  FT_TRY(push_table_rows(c, dirty, s));
  c->last_stream = s;
  return FT_OK;
}

extern "C" ft_status ft_expert_cache_resize(ft_ctx* c, int64_t new_budget) {
  NvtxRange nvtx_range("ft_expert_cache_resize");
  if (!c) return fail(FT_ERR_INVALID, "ctx is NULL");
  if (new_budget < 0) return fail(FT_ERR_INVALID, "negative budget");
  if (!c->cache_on) return fail(FT_ERR_INVALID, "context has no expert cache");
  CUDA_TRY(cudaDeviceSynchronize());
  for (auto& kv : c->pending) c->spare_miss_events.push_back(kv.second);  // every copy has landed
  c->pending.clear();
  int64_t cap = new_budget / c->stride;
  if ((size_t)cap * c->stride > c->va_size) return fail(FT_ERR_NO_SPACE, "budget larger than the reserved arena");
  const int64_t old_cap = c->lru.capacity;
  // grow: map the physical memory first, so that the capacity only ever
  // covers mapped slots (a failed map leaves the old capacity in force)
  if (cap > old_cap) FT_TRY(arena_map(c, cap));
  if (cap < old_cap) {
    while ((int64_t)c->lru.map.size() > cap) evict_one(c, {});
    // survivors in slots >= cap move down to the lowest free slots, ascending
    std::vector<std::pair<int32_t, int64_t>> movers;
    for (auto& kv : c->lru.map)
      if (kv.second.first >= cap) movers.push_back({kv.second.first, kv.first});
    std::sort(movers.begin(), movers.end());
    for (auto& mv : movers) {
      int32_t from = mv.first;
      int32_t to = -1;
      for (int64_t s2 = 0; s2 < cap; s2++)
        if (!c->lru.slot_used[s2]) {
          to = (int32_t)s2;
          break;
        }
      CUDA_TRY(cudaMemcpyAsync(slot_ptr(c, to), slot_ptr(c, from), (size_t)c->lay.used, cudaMemcpyDeviceToDevice,
                               c->copy_stream));
      c->lru.slot_used[from] = 0;
      c->lru.slot_used[to] = 1;
      c->lru.map[mv.second].first = to;
      int layer = (int)(mv.second / c->d.n_experts), e = (int)(mv.second % c->d.n_experts);
      c->h_eptr_cache[(size_t)layer * c->n_blobs + e] = slot_ptr(c, to);
      record(c, FT_EV_MOVE, layer, e, to, from);
      c->stats.moves++;
    }
    CUDA_TRY(cudaStreamSynchronize(c->copy_stream));
  }
  c->lru.set_capacity(cap);
  for (int64_t s2 = cap; s2 < (int64_t)c->lru.slot_used.size(); s2++) c->lru.slot_used[s2] = 0;
  c->stats.capacity_slots = cap;
  c->stats.used_slots = (int64_t)c->lru.map.size();
  // shrink: unmap only after the survivors moved below the new capacity
  if (cap < old_cap) FT_TRY(arena_map(c, cap));
  CUDA_TRY(cudaMemcpy(c->d_eptr_cache, c->h_eptr_cache, (size_t)c->d.n_layers * c->n_blobs * sizeof(void*),
                      cudaMemcpyHostToDevice));
  return FT_OK;
}

extern "C" ft_status ft_cache_trace(ft_ctx* c, ft_cache_event* buf, int64_t cap, int64_t* n) {
  if (!c || !n || (cap > 0 && !buf)) return fail(FT_ERR_INVALID, "NULL argument");
  int64_t m = std::min<int64_t>(cap, (int64_t)c->trace.size());
  if (m > 0) memcpy(buf, c->trace.data(), (size_t)m * sizeof(ft_cache_event));
  *n = m;
  const bool over = (int64_t)c->trace.size() > cap;
  const int64_t dropped = c->trace_dropped;
  c->trace.clear();
  c->trace_dropped = 0;
  if (dropped > 0)
    return fail(FT_ERR_NO_SPACE, "%lld events were dropped: the trace holds at most %lld between reads",
                (long long)dropped, (long long)kTraceMaxEvents);
  if (over) return fail(FT_ERR_NO_SPACE, "trace had more events than cap");
  return FT_OK;
}

extern "C" ft_status ft_cache_stats_get(ft_ctx* c, ft_cache_stats* out, int32_t reset) {
  if (!c || !out) return fail(FT_ERR_INVALID, "NULL argument");
  if (!c->copy_timing.empty()) {
    CUDA_TRY(cudaStreamSynchronize(c->copy_stream));
    fold_copy_timing(c);
  }
  *out = c->stats;
  if (reset) {
    int64_t cap = c->stats.capacity_slots, used = c->stats.used_slots, mapped = c->stats.mapped_bytes;
    c->stats = ft_cache_stats{};
    c->stats.capacity_slots = cap;
    c->stats.used_slots = used;
    c->stats.mapped_bytes = mapped;
  }
  return FT_OK;
}

// ---------------------------------------------------------------------------
// prefetch
// ---------------------------------------------------------------------------
extern "C" ft_status ft_prefetch_layer(ft_ctx* c, int32_t layer, void* compute_stream) {
  NvtxRange nvtx_range("ft_prefetch_layer");
  if (!c) return fail(FT_ERR_INVALID, "ctx is NULL");
  if (layer < 0 || layer >= c->d.n_layers) return fail(FT_ERR_INVALID, "layer %d out of range", layer);
  if (!c->host_layers[layer]) return fail(FT_ERR_NOT_FOUND, "layer %d has no host pool", layer);
  (void)compute_stream;
  const int b = layer & 1;
  const size_t bytes = (size_t)c->n_blobs * c->stride;
  if (!c->d_stage[b]) {
    // both allocations, or neither: a later call must not find a buffer
    // without its pointer table
    uint8_t* stage = nullptr;
    const uint8_t** table = nullptr;
    std::vector<const uint8_t*> tab(c->n_blobs);
    if (cudaMalloc((void**)&stage, bytes) != cudaSuccess ||
        cudaMalloc((void**)&table, c->n_blobs * sizeof(void*)) != cudaSuccess) {
      cudaFree(stage);
      cudaGetLastError();
      return fail(FT_ERR_CUDA, "staging buffer of %zu bytes", bytes);
    }
    for (int e = 0; e < c->n_blobs; e++) tab[e] = stage + (size_t)e * c->stride;
    if (cudaMemcpy(table, tab.data(), c->n_blobs * sizeof(void*), cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaFree(stage);
      cudaFree(table);
      return fail(FT_ERR_CUDA, "staging pointer table");
    }
    c->d_stage[b] = stage;
    c->d_eptr_stage[b] = table;
  }
  // reuse only after the last forward that read this buffer is done
  CUDA_TRY(cudaStreamWaitEvent(c->copy_stream, c->ev_done[b], 0));
  CUDA_TRY(cudaMemcpyAsync(c->d_stage[b], c->host_layers[layer], bytes, cudaMemcpyHostToDevice, c->copy_stream));
  CUDA_TRY(cudaEventRecord(c->ev_landed[b], c->copy_stream));
  c->stage_layer[b] = layer;
  c->prefetch_bytes += (int64_t)bytes;
  return FT_OK;
}

// ---------------------------------------------------------------------------
// layer forward
// ---------------------------------------------------------------------------
static DecodeArgs decode_args(ft_ctx* c, const uint16_t* x, const Route* rec, int T, const uint8_t* const* eptr,
                              uint16_t* out) {
  DecodeArgs a{};
  a.x = x;
  a.rec = rec;
  a.T = T;
  a.H = c->d.hidden;
  a.I = c->d.inter;
  a.E = c->d.n_experts;
  a.k = c->d.top_k;
  a.n_shared = c->d.n_shared;
  a.max_units = std::min(a.E, T * a.k);
  a.eptr = eptr;
  a.lay = c->lay;
  a.h = c->d_h;
  a.y = c->d_y;
  a.out = out;
  a.counters = c->d_counters;
  a.status = c->d_status;
  return a;
}

static RouteArgs route_args(ft_ctx* c, const float* logits, int T, int n_layers, uint32_t flags, Route* rec) {
  RouteArgs r{};
  r.logits = logits;
  r.T = T;
  r.E = c->d.n_experts;
  r.k = c->d.top_k;
  r.renorm = (flags & FT_ROUTE_RENORM) ? 1 : 0;
  r.n_layers = n_layers;
  r.rec = rec;
  r.ids_out = c->d_ids;
  r.w_out = c->d_w;
  r.status = c->d_status;
  return r;
}

extern "C" ft_status ft_moe_layer_forward(ft_ctx* c, int32_t layer, const void* x, int64_t T,
                                          const float* router_w, const float* logits_override, void* out,
                                          uint32_t flags, void* stream) {
  NvtxRange nvtx_range("ft_moe_layer_forward");
  if (!c || !out || (!x && T > 0)) return fail(FT_ERR_INVALID, "NULL argument");
  if (layer < 0 || layer >= c->d.n_layers) return fail(FT_ERR_INVALID, "layer %d out of range", layer);
  if (T < 0 || T > c->max_tokens) return fail(FT_ERR_INVALID, "T=%lld outside [0, max_tokens=%d]", (long long)T, c->max_tokens);
  if (!logits_override && !router_w) return fail(FT_ERR_INVALID, "need router_w or logits_override");
  if (x == out) return fail(FT_ERR_INVALID, "out must not alias x");
  if (!aligned16(x) || !aligned16(out) || !aligned16(router_w) || !aligned16(logits_override))
    return fail(FT_ERR_INVALID, "x, out, router_w and logits must start on a 16-byte boundary");
  // prefill path: FT_ACT_MXFP4 (MXFP4 weights) or FT_ACT_NVFP4 (NVFP4 weights)
  const bool nv = (flags & FT_ACT_NVFP4) != 0;
  const bool pf = nv || (flags & FT_ACT_MXFP4) != 0;
  if (nv && (flags & FT_ACT_MXFP4)) return fail(FT_ERR_INVALID, "FT_ACT_MXFP4 and FT_ACT_NVFP4 exclude each other");
  if (pf && (c->d.hidden % 256 || c->d.inter % 256))
    return fail(FT_ERR_INVALID, "the prefill path needs hidden and inter to be multiples of 256");
  if (pf && !nv && c->d.weight_format != FT_FMT_MXFP4)
    return fail(FT_ERR_INVALID, "FT_ACT_MXFP4 (prefill) takes MXFP4 weights only");
  if (nv && c->d.weight_format != FT_FMT_NVFP4)
    return fail(FT_ERR_INVALID, "FT_ACT_NVFP4 (prefill) takes NVFP4 weights only");
  if (!pf && T > c->decode_max_t)
    return fail(FT_ERR_INVALID, "decode GEMV path takes T <= %d (use FT_ACT_MXFP4 for prefill)", c->decode_max_t);
  if (!pf && !decode_supported(c->d.hidden, c->d.inter, c->d.weight_format))
    return fail(FT_ERR_INVALID, "decode GEMV path takes hidden and inter up to 16384 (use FT_ACT_MXFP4)");
  if (T == 0) return FT_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const int H = c->d.hidden, E = c->d.n_experts, k = c->d.top_k, Ti = (int)T;

  // 1-3: logits, then routing.  The decode kernels route inside every CTA;
  // the separate top-k / permutation kernels run for prefill, and top-k alone
  // for the cache path, whose host LRU needs the ids first.
  const float* logits = logits_override;
  if (!logits) {
    KTimer kt(c, FT_K_ROUTER_LOGITS, s);
    CUDA_TRY(launch_router_logits((const uint16_t*)x, router_w, Ti, H, E, c->d_logits, s));
    logits = c->d_logits;
  }
  Route* rec = c->d_routes + layer;
  if (pf) {
    KTimer kt(c, FT_K_TOPK, s);
    CUDA_TRY(launch_topk(logits, Ti, E, k, (flags & FT_ROUTE_RENORM) ? 1 : 0, c->d_ids, c->d_w, c->d_status, s));
  } else {
    KTimer kt(c, FT_K_TOPK, s);
    CUDA_TRY(launch_route(route_args(c, logits, Ti, 1, flags, rec), s));
  }
  if (pf) {
    KTimer kt(c, FT_K_PERMUTE, s);
    CUDA_TRY(launch_permute(c->d_ids, Ti * k, E, c->d_offs, c->d_perm, c->d_inv, c->d_active, c->d_nact,
                            c->d_pad_offs, c->d_status, s));
  }

  // 4: weight source.  Prefill (MXFP4) reads resident or staged layers and
  // never touches the cache; decode reads resident layers or the cache.
  const uint8_t* const* eptr = nullptr;
  std::vector<int> miss_units;  // cache path: units whose blobs are still being copied, in copy order
  int n_routed_units = 0;
  bool step_timed = false;      // cache path: this step's copies have a timing entry
  bool cache_layer = false;     // cache path taken
  std::vector<int> step_set;    // cache path: the step's distinct experts
  const uint8_t* pool = nullptr;
  int stage_buf = -1;
  if (c->resident[layer]) {
    eptr = c->d_eptr_res + (size_t)layer * c->n_blobs;
    pool = c->resident[layer];
  } else if (pf) {
    if (c->stage_layer[layer & 1] != layer)
      return fail(FT_ERR_NOT_FOUND, "prefill of layer %d: not resident and not prefetched", layer);
    stage_buf = layer & 1;
    CUDA_TRY(cudaStreamWaitEvent(s, c->ev_landed[stage_buf], 0));
    eptr = c->d_eptr_stage[stage_buf];
    pool = c->d_stage[stage_buf];
  } else if (c->cache_on && c->host_layers[layer]) {
    CUDA_TRY(cudaMemcpyAsync(c->h_ids, c->d_ids, (size_t)Ti * k * sizeof(int32_t), cudaMemcpyDeviceToHost, s));
    CUDA_TRY(cudaMemcpyAsync(c->h_status, c->d_status, sizeof(int), cudaMemcpyDeviceToHost, s));
    CUDA_TRY(cudaEventRecord(c->ev_ids, s));
    // timing anchor of the step: everything below comes after it
    cudaEvent_t ref = copy_event(c);
    CUDA_TRY(cudaEventRecord(ref, s));
    const ft_status ws = wait_event(c->ev_ids, "routing ids", c->host_wait_s);
    if (ws != FT_OK) {
      c->spare_events.push_back(ref);
      return ws;
    }
    if (*c->h_status) {
      c->spare_events.push_back(ref);
      int st = *c->h_status;
      CUDA_TRY(cudaMemsetAsync(c->d_status, 0, sizeof(int), s));
      return status_to_ft(st);
    }
    std::vector<int> S(c->h_ids, c->h_ids + (size_t)Ti * k);
    for (int e : S)
      if (e < 0 || e >= E) {
        c->spare_events.push_back(ref);
        return fail(FT_ERR_INVALID, "expert id %d out of range", e);
      }
    std::sort(S.begin(), S.end());
    S.erase(std::unique(S.begin(), S.end()), S.end());
    std::vector<int> dirty{layer};
    bool any_miss = false;
    {
      NvtxRange step_range("cache_step");
      ft_status cs = cache_step(c, layer, S, any_miss, dirty, &miss_units, ref);
      if (!any_miss && cs == FT_OK) ref = nullptr;  // returned to the pool by cache_step
      if (cs != FT_OK) {
        for (cudaEvent_t e : c->miss_events) c->spare_miss_events.push_back(e);
        c->miss_events.clear();
        return cs;
      }
    }
    FT_TRY(push_table_rows(c, dirty, s));
    eptr = c->d_eptr_cache + (size_t)layer * c->n_blobs;
    if (!miss_units.empty() && (flags & FT_CACHE_SERIAL)) {
      // the serial order, for comparison: every copy lands before any expert runs
      for (cudaEvent_t e : c->miss_events) CUDA_TRY(cudaStreamWaitEvent(s, e, 0));
      miss_units.clear();
    }
    n_routed_units = (int)S.size();
    step_timed = any_miss;
    cache_layer = true;
    step_set = S;
  } else {
    return fail(FT_ERR_NOT_FOUND, "layer %d is neither resident nor cached", layer);
  }

  // 5: experts and combine
  if (!pf && !miss_units.empty()) {
    // cache path with misses: the resident experts (hits and the shared
    // experts) run at once, while the misses' copies are in flight; each
    // missed expert runs after its own copy ([no] experts fetched over PCIe;
    // the copies overlap the compute of the experts already resident)
    DecodeArgs a = decode_args(c, (const uint16_t*)x, rec, Ti, eptr, (uint16_t*)out);
    std::vector<char> is_miss((size_t)n_routed_units, 0);
    for (int u : miss_units) is_miss[u] = 1;
    a.n_sel = 0;
    for (int u = 0; u < n_routed_units; u++)
      if (!is_miss[u]) a.sel[a.n_sel++] = (uint16_t)u;
    for (int sx = 0; sx < c->d.n_shared; sx++) a.sel[a.n_sel++] = (uint16_t)(a.max_units + sx);
    ft_ctx::StepTiming* stp = step_timed ? &c->copy_timing.back() : nullptr;
    if (a.n_sel > 0) {
      if (stp) {
        stp->h0 = copy_event(c);
        stp->h1 = copy_event(c);
        CUDA_TRY(cudaEventRecord(stp->h0, s));
      }
      {
        KTimer kt(c, FT_K_GATE_UP, s);
        CUDA_TRY(launch_dec_gate_up(a, false, s));
      }
      {
        KTimer kt(c, FT_K_DOWN_COMBINE, s);
        CUDA_TRY(launch_dec_down(a, true, s));
      }
      if (stp) CUDA_TRY(cudaEventRecord(stp->h1, s));
    }
    for (size_t mi = 0; mi < miss_units.size(); mi++) {
      CUDA_TRY(cudaStreamWaitEvent(s, c->miss_events[mi], 0));
      a.n_sel = 1;
      a.sel[0] = (uint16_t)miss_units[mi];
      {
        KTimer kt(c, FT_K_GATE_UP, s);
        CUDA_TRY(launch_dec_gate_up(a, false, s));
      }
      {
        KTimer kt(c, FT_K_DOWN_COMBINE, s);
        CUDA_TRY(launch_dec_down(a, true, s));
      }
    }
    // the waits above hold the events' current records: they can be reused
    for (cudaEvent_t e : c->miss_events) c->spare_miss_events.push_back(e);
    c->miss_events.clear();
  } else if (!pf) {
    for (cudaEvent_t e : c->miss_events) c->spare_miss_events.push_back(e);
    c->miss_events.clear();
    DecodeArgs a = decode_args(c, (const uint16_t*)x, rec, Ti, eptr, (uint16_t*)out);
    {
      KTimer kt(c, FT_K_GATE_UP, s);
      CUDA_TRY(launch_dec_gate_up(a, false, s));
    }
    {
      KTimer kt(c, FT_K_DOWN_COMBINE, s);
      CUDA_TRY(launch_dec_down(a, true, s));
    }
  } else {
    if (ensure_prefill_scratch(c->pf, c->d, c->max_tokens) != FT_OK)
      return fail(FT_ERR_CUDA, "prefill scratch allocation failed");
    PrefillArgs a{};
    a.x = (const uint16_t*)x;
    a.T = Ti;
    a.H = H;
    a.I = c->d.inter;
    a.E = E;
    a.k = k;
    a.n_shared = c->d.n_shared;
    a.ids = c->d_ids;
    a.w = c->d_w;
    a.offs = c->d_offs;
    a.perm = c->d_perm;
    a.inv = c->d_inv;
    a.pad_offs = c->d_pad_offs;
    a.eptr = eptr;
    a.pool = pool;
    a.lay = c->lay;
    a.out = (uint16_t*)out;
    a.status = c->d_status;
    CUDA_TRY(launch_shared_segments(c->d_pad_offs, E, Ti, c->d.n_shared, s));
    {
      KTimer kt(c, FT_K_QUANT_X, s);
      CUDA_TRY(launch_quant_x(c->pf, a, s));
    }
    {
      KTimer kt(c, FT_K_GEMM_GATE_UP, s);
      CUDA_TRY(launch_prefill_gemm(c->pf, a, 0, s));
    }
    if (nv) {
      KTimer kt(c, FT_K_QUANT_H, s);
      CUDA_TRY(launch_quant_h(c->pf, a, s));
    }
    {
      KTimer kt(c, FT_K_GEMM_DOWN, s);
      CUDA_TRY(launch_prefill_gemm(c->pf, a, 1, s));
    }
    {
      KTimer kt(c, FT_K_COMBINE, s);
      CUDA_TRY(launch_prefill_combine(c->pf, a, s));
    }
  }
  if (stage_buf >= 0) CUDA_TRY(cudaEventRecord(c->ev_done[stage_buf], s));
  c->last_stream = s;
  // cache path: count the step's experts; the next layer's prefetch follows
  // the step's own copies on the copy stream
  if (cache_layer) FT_TRY(prefetch_next(c, layer, step_set));
  return FT_OK;
}

// ---------------------------------------------------------------------------
// per-kernel timing
// ---------------------------------------------------------------------------
static void drop_marks(ft_ctx* c, bool graph_too) {
  for (auto& m : c->tmarks) {
    cudaEventDestroy(m.second.first);
    cudaEventDestroy(m.second.second);
  }
  c->tmarks.clear();
  if (!graph_too) return;
  for (auto& m : c->gmarks) {
    cudaEventDestroy(m.second.first);
    cudaEventDestroy(m.second.second);
  }
  c->gmarks.clear();
}

extern "C" ft_status ft_kernel_timing_enable(ft_ctx* c, int32_t on) {
  if (!c) return fail(FT_ERR_INVALID, "ctx is NULL");
  CUDA_TRY(cudaDeviceSynchronize());
  drop_marks(c, true);
  for (int i = 0; i < FT_K_COUNT; i++) {
    c->tms[i] = 0;
    c->tlaunch[i] = 0;
  }
  c->timing = on != 0;
  return FT_OK;
}

extern "C" ft_status ft_kernel_timing_read(ft_ctx* c, double* ms, int64_t* launches, int32_t n) {
  if (!c || !ms || !launches || n < 0) return fail(FT_ERR_INVALID, "bad argument");
  CUDA_TRY(cudaDeviceSynchronize());
  for (auto* v : {&c->tmarks, &c->gmarks})
    for (auto& m : *v) {
      float t = 0.f;
      if (cudaEventElapsedTime(&t, m.second.first, m.second.second) != cudaSuccess) {
        cudaGetLastError();  // a captured mark whose graph has not run yet
        continue;
      }
      c->tms[m.first] += t;
      c->tlaunch[m.first] += 1;
    }
  drop_marks(c, false);
  for (int i = 0; i < n && i < FT_K_COUNT; i++) {
    ms[i] = c->tms[i];
    launches[i] = c->tlaunch[i];
  }
  return FT_OK;
}

// ---------------------------------------------------------------------------
// stacked decode over consecutive resident layers
// ---------------------------------------------------------------------------
extern "C" ft_status ft_moe_stack_forward(ft_ctx* c, int32_t first_layer, int32_t n_layers, const void* x, int64_t T,
                                          const float* logits, void* out, uint32_t flags, void* stream) {
  NvtxRange nvtx_range("ft_moe_stack_forward");
  if (!c || !x || !out || !logits) return fail(FT_ERR_INVALID, "NULL argument");
  if (n_layers <= 0 || first_layer < 0 || first_layer + n_layers > c->d.n_layers)
    return fail(FT_ERR_INVALID, "layers [%d, %d) outside [0, %d)", first_layer, first_layer + n_layers, c->d.n_layers);
  if (T < 0 || T > c->decode_max_t) return fail(FT_ERR_INVALID, "T=%lld outside [0, %d]", (long long)T, c->decode_max_t);
  if (!decode_supported(c->d.hidden, c->d.inter, c->d.weight_format))
    return fail(FT_ERR_INVALID, "decode kernels take hidden and inter up to 16384");
  if (flags & (FT_ACT_MXFP4 | FT_ACT_NVFP4))
    return fail(FT_ERR_INVALID, "the stacked forward is the decode path (FT_ACT_BF16)");
  if (x == out) return fail(FT_ERR_INVALID, "out must not alias x");
  if (!aligned16(x) || !aligned16(out) || !aligned16(logits))
    return fail(FT_ERR_INVALID, "x, out and logits must start on a 16-byte boundary");
  for (int l = first_layer; l < first_layer + n_layers; l++)
    if (!c->resident[l]) return fail(FT_ERR_STATE, "layer %d is not resident", l);
  if (T == 0) return FT_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const int Ti = (int)T;
  const int H = c->d.hidden, I = c->d.inter;
  const bool layerwise = (flags & FT_STACK_LAYERWISE) != 0;
  // one or two tokens: the dataflow kernel (tagged h and x, down tiles over
  // every unit); three or four tokens: the dataflow kernel in waves of two
  // (the tokens of a MoE layer do not interact, and each wave computes its
  // tokens' bits as the per-layer path does); else, or with
  // FT_STACK_COUNTERS, the counter-synchronised persistent kernel; else two
  // kernels per layer
  const int wave = Ti <= 2 ? Ti : 2;
  const FlowGeom fg = flow_geometry(H, I, wave, c->d.top_k, c->d.n_shared, c->d.n_experts, n_layers,
                                    c->d.weight_format);
  const bool flow = !layerwise && !(flags & FT_STACK_COUNTERS) && c->d_tagged != nullptr && fg.ok && Ti <= 4;
  // the counter-synchronised kernel computes MXFP4 weights only
  const bool persistent = !layerwise && !flow && c->d_sync != nullptr && c->d.weight_format == FT_FMT_MXFP4 &&
                          stack_supported(H, I, n_layers);
  if (flow) {
    int dev = 0, nsm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int E = c->d.n_experts, k = c->d.top_k;
    for (int t0 = 0; t0 < Ti; t0 += wave) {
      const int Tw = std::min(wave, Ti - t0);
      const FlowGeom fw = Tw == wave ? fg : flow_geometry(H, I, Tw, k, c->d.n_shared, E, n_layers, c->d.weight_format);
      // the wave's routing records, from its rows of every layer's logits
      {
        KTimer kt(c, FT_K_TOPK, s);
        RouteArgs ra = route_args(c, logits + (size_t)t0 * E, Tw, n_layers, flags, c->d_routes + first_layer);
        ra.layer_stride = (int64_t)Ti * E;
        ra.ids_out = c->d_ids + (size_t)t0 * k;
        ra.w_out = c->d_w + (size_t)t0 * k;
        ra.epoch = c->d_epoch;
        ra.tagged = c->d_tagged;
        ra.tagged_words = c->tagged_words;
        CUDA_TRY(launch_route(ra, s));
      }
      FlowArgs a{};
      a.x0 = (const uint16_t*)x + (size_t)t0 * H;
      a.out = (uint16_t*)out + (size_t)t0 * H;
      a.rec = c->d_routes + first_layer;
      a.eptr = c->d_eptr_res + (size_t)first_layer * c->n_blobs;
      a.n_layers = n_layers;
      a.n_blobs = c->n_blobs;
      a.T = Tw;
      a.H = H;
      a.I = I;
      a.E = E;
      a.k = k;
      a.n_shared = c->d.n_shared;
      a.lay = c->lay;
      a.h_tagged = c->d_h_tagged;
      a.x_tagged = c->d_x_tagged;
      a.epoch = c->d_epoch;
      a.rows_cap = fw.rows_cap;
      a.status = c->d_status;
      a.timeline = c->timeline && c->timeline_words >= (int64_t)n_layers * nsm * 8 ? c->timeline : nullptr;
      KTimer kt(c, FT_K_DEC_STACK, s);
      CUDA_TRY(launch_dec_flow(a, s));
    }
    c->last_stream = s;
    return FT_OK;
  }
  // all layers' routing records in one launch (their logits are inputs); it
  // also zeroes the counter-synchronised kernel's counters of those layers
  {
    KTimer kt(c, FT_K_TOPK, s);
    RouteArgs ra = route_args(c, logits, Ti, n_layers, flags, c->d_routes + first_layer);
    if (persistent) {
      ra.sync = c->d_sync;
      ra.sync_stride = c->sync_stride;
    }
    CUDA_TRY(launch_route(ra, s));
  }
  if (persistent) {
    StackArgs a{};
    a.x0 = (const uint16_t*)x;
    a.out = (uint16_t*)out;
    a.xbuf[0] = c->d_xbuf[0];
    a.xbuf[1] = c->d_xbuf[1];
    a.rec = c->d_routes + first_layer;
    a.eptr = c->d_eptr_res + (size_t)first_layer * c->n_blobs;
    a.n_layers = n_layers;
    a.n_blobs = c->n_blobs;
    a.T = Ti;
    a.H = c->d.hidden;
    a.I = c->d.inter;
    a.E = c->d.n_experts;
    a.k = c->d.top_k;
    a.n_shared = c->d.n_shared;
    a.lay = c->lay;
    a.h = c->d_h;
    a.y = c->d_y;
    a.sync = c->d_sync;
    a.sync_stride = c->sync_stride;
    a.status = c->d_status;
    KTimer kt(c, FT_K_DEC_STACK, s);
    CUDA_TRY(launch_dec_stack(a, s));
    c->last_stream = s;
    return FT_OK;
  }
  const uint16_t* cur = (const uint16_t*)x;
  for (int i = 0; i < n_layers; i++) {
    const int l = first_layer + i;
    uint16_t* dst = (i == n_layers - 1) ? (uint16_t*)out : c->d_xbuf[i & 1];
    DecodeArgs a = decode_args(c, cur, c->d_routes + l, Ti, c->d_eptr_res + (size_t)l * c->n_blobs, dst);
    // after the first layer, a layer's gate/up starts staging its weights
    // while the previous layer finishes: its routing record and pointer
    // table were complete before the first layer's gate/up started
    {
      KTimer kt(c, FT_K_GATE_UP, s);
      CUDA_TRY(launch_dec_gate_up(a, i > 0 && !c->timing, s));
    }
    {
      KTimer kt(c, FT_K_DOWN_COMBINE, s);
      CUDA_TRY(launch_dec_down(a, true, s));
    }
    cur = dst;
  }
  c->last_stream = s;
  return FT_OK;
}

extern "C" ft_status ft_last_routing(ft_ctx* c, int32_t* ids, float* w, int64_t n, void* stream) {
  if (!c || !ids || !w) return fail(FT_ERR_INVALID, "NULL argument");
  if (n < 0 || n > (int64_t)c->max_tokens * c->d.top_k) return fail(FT_ERR_INVALID, "n out of range");
  CUDA_TRY(cudaMemcpyAsync(ids, c->d_ids, (size_t)n * sizeof(int32_t), cudaMemcpyDefault, (cudaStream_t)stream));
  CUDA_TRY(cudaMemcpyAsync(w, c->d_w, (size_t)n * sizeof(float), cudaMemcpyDefault, (cudaStream_t)stream));
  return FT_OK;
}

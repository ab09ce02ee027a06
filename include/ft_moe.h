/*
 * ft_moe.h — C ABI of libftmoe.so: one MoE layer forward pass with a GPU
 * expert cache over a pinned host expert pool, for NVIDIA B200 (sm_100a).
 *
 * Method: the FreeToken serving engine as described in its public write-ups.
 * Citations name the page and its section (or paragraph topic):
 *   [hu]  aiforradalom.hu, "Egyetlen munkaállomás-GPU-n futtatja a 753
 *         milliárdos GLM-5.2 modellt a FreeToken", section "A Mixture-of-Experts
 *         (MoE) kihívásai és a FreeToken megoldásai"
 *   [no]  jansverre.net, "FreeToken GLM-5.2 en GPU", sections "Hva er
 *         FreeToken?" and "Hvorfor er båndbredden viktigere enn antall kjerner?"
 *   [fa]  aipolix.com, "FreeToken مدلهای عظیم MoE را روی GPUهای مصرفی اجرا
 *         میکند", paragraphs on bandwidth-adaptive execution, on
 *         semantic-aware caching and on elastic memory management
 *
 * Conventions
 *   - Every call returns ft_status; nothing throws across the ABI.  On error
 *     ft_last_error() gives a message (thread-local, valid until the next call
 *     from the same thread).
 *   - "dev" pointers are CUDA device pointers owned by the caller; "host"
 *     pointers are host memory owned by the caller.  Streams are cudaStream_t
 *     values passed as void* (NULL = the legacy default stream).
 *   - Kernels run asynchronously on the given stream.  Errors that only the
 *     device can see (a NaN or +inf logit, an expert id out of range, a bounded
 *     device wait that gave up) set a status word in the context; they are
 *     returned by ft_sync_status() and by the next call that synchronises
 *     with the host (the cache path of ft_moe_layer_forward does).
 *   - Sizes are int64_t, ids int32_t.  Calls on one context are not
 *     thread-safe and must be ordered by the caller (one compute stream).
 *
 * Expert weight format (one "blob" per expert, stride ft_blob_stride()):
 *   codes, row-major, K contiguous, two e2m1 codes per byte (element 2i in the
 *   low nibble): Wg [I][H], Wu [I][H], Wd [H][I]; then UE8M0 block scales (one
 *   byte per 32 elements along K) of Wg, Wu, Wd, each region tiled in 512-byte
 *   atoms of 128 rows x 4 blocks (row r at byte (r%32)*16 + ((r%128)/32)*4 +
 *   block%4; atoms along K first); zero padding to a multiple of 256 bytes.
 *   A layer holds n_experts routed blobs followed by n_shared shared blobs.
 *   MXFP4 = e2m1 elements with per-32 UE8M0 scales ([no] "MXFP4";
 *   [hu] FP4 expert pool).
 */
#ifndef FT_MOE_H
#define FT_MOE_H

#include <stdint.h>

#if defined(__GNUC__)
#define FT_API __attribute__((visibility("default")))
#else
#define FT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FT_OK = 0,
  FT_ERR_INVALID = 1,    /* bad argument or shape */
  FT_ERR_CUDA = 2,       /* a CUDA runtime / driver call failed */
  FT_ERR_NO_SPACE = 3,   /* cache capacity below the experts one step needs */
  FT_ERR_TIMEOUT = 4,    /* a bounded host or device wait gave up */
  FT_ERR_NOT_FOUND = 5,  /* key not resident / layer not staged */
  FT_ERR_NONFINITE = 6,  /* NaN or +inf router logit, or a row with no finite logit */
  FT_ERR_STATE = 7       /* call not valid in the context's current state */
} ft_status;

typedef struct ft_ctx ft_ctx;

typedef struct {
  int32_t hidden;             /* H, multiple of 128 */
  int32_t inter;              /* I, expert intermediate size, multiple of 128 */
  int32_t n_experts;          /* E routed experts per layer, <= 1024 */
  int32_t top_k;              /* k experts per token, <= 16 and <= E */
  int32_t n_layers;           /* L */
  int32_t n_shared;           /* always-on shared experts per layer (weight 1), 0 or 1 */
  int64_t cache_budget_bytes; /* GPU expert-cache budget (0 = no cache) */
  int32_t max_tokens;         /* largest T any forward call passes; sizes scratch */
  int32_t weight_format;      /* FT_FMT_MXFP4 (0), FT_FMT_NVFP4 or FT_FMT_BF16 */
} ft_model_desc;

/* Expert weight formats ([no] "Hvor raskt kjører modellene?": MXFP4 for
 * DeepSeek-V4-Flash, BF16 and NVFP4 builds of Qwen3.6-35B-A3B).  Blob layouts
 * (each matrix K-contiguous, padded to a multiple of 256 bytes):
 *   MXFP4  as described above (ft_blob_stride);
 *   NVFP4  the same e2m1 code regions; then E4M3 block scales (one per 16
 *          elements along K; no infinities, S.1111.111 is NaN) in the same
 *          128-row x 4-block atoms; then the fp32 scales of Wg, Wu, Wd and 4
 *          zero bytes.  A weight is code value x block scale x matrix scale.
 *   BF16   Wg [I][H], Wu [I][H], Wd [H][I] as little-endian bf16.
 * The decode paths (FT_ACT_BF16) take every format; the prefill path takes
 * MXFP4 weights with FT_ACT_MXFP4 and NVFP4 weights with FT_ACT_NVFP4. */
#define FT_FMT_MXFP4 0
#define FT_FMT_NVFP4 1
#define FT_FMT_BF16  2

/* forward / route flags */
#define FT_ROUTE_RENORM 1u    /* renormalise the k softmax weights to sum 1 (default on) */
#define FT_ACT_BF16     0u    /* decode: bf16 activations, fp32 h, FP4 GEMV on CUDA cores */
#define FT_ACT_MXFP4    2u    /* prefill: x and h quantised to MXFP4, tcgen05 grouped GEMM */
#define FT_STACK_LAYERWISE 4u /* ft_moe_stack_forward: two kernels per layer, not a persistent kernel */
#define FT_STACK_COUNTERS  8u /* ft_moe_stack_forward: the counter-synchronised persistent kernel, not the dataflow one */
#define FT_CACHE_SERIAL   16u /* cache path: every miss copy lands before any expert runs (for comparison) */
#define FT_ACT_NVFP4      32u /* prefill with NVFP4 weights: x and h quantised to NVFP4, grouped GEMM on
                                 tcgen05 kind::mxf4nvf4 (see ft_quantize_nvfp4 for the quantiser) */

/* cache trace events */
#define FT_EV_HIT   0
#define FT_EV_MISS  1
#define FT_EV_EVICT 2
#define FT_EV_MOVE  3
#define FT_EV_PREFETCH 4   /* inserted ahead of use by ft_cache_prefetch's policy */
typedef struct {
  int32_t kind;      /* FT_EV_* */
  int32_t layer;
  int32_t expert;
  int32_t slot;      /* slot after the event (the freed slot for EVICT) */
  int32_t from_slot; /* old slot for MOVE, -1 otherwise */
} ft_cache_event;

typedef struct {
  int64_t hits, misses, evictions, moves;
  int64_t h2d_bytes;          /* bytes fetched from the host pool by misses */
  double  h2d_ms;             /* copy-stream time of those fetches (CUDA events) */
  double  hit_ms;             /* time of the resident experts' kernels of steps with misses */
  double  overlap_ms;         /* part of hit_ms that ran while that step's copies were in flight */
  int64_t capacity_slots, used_slots;
  int64_t mapped_bytes;       /* physical memory mapped under the slot arena */
  int64_t prefetches;         /* keys inserted by the next-layer prefetch */
  int64_t prefetch_hits;      /* prefetched keys later hit (each counted once) */
  int64_t prefetch_bytes;     /* bytes copied by those prefetches */
} ft_cache_stats;

/* ---------------------------------------------------------------------- */
/* format                                                                  */
/* ---------------------------------------------------------------------- */

/* Bytes per expert blob for hidden H and intermediate I (>= 0; -1 on bad shape).
 * Equals 3*H*I*17/32 when the scale regions fill whole atoms. */
FT_API int64_t ft_blob_stride(int32_t hidden, int32_t inter);

/* Byte offsets of the regions of a blob: out[0..7] = Wg, Wu, Wd codes,
 * Wg, Wu, Wd scales, used bytes, stride.  FT_ERR_INVALID on a bad shape. */
FT_API ft_status ft_blob_layout(int32_t hidden, int32_t inter, int64_t out[8]);

/* The same for weight format fmt (FT_FMT_*): out[0..7] as ft_blob_layout
 * (for BF16 the scale offsets equal the used bytes), out[8] the NVFP4 matrix
 * scales' offset (-1 otherwise).  FT_ERR_INVALID on a bad shape or format. */
FT_API ft_status ft_blob_layout_format(int32_t hidden, int32_t inter, int32_t fmt, int64_t out[9]);

/* Message of the last error on this thread ("" if none). */
FT_API const char* ft_last_error(void);

/* ---------------------------------------------------------------------- */
/* context                                                                 */
/* ---------------------------------------------------------------------- */

/* Alignment: every device buffer passed to the calls below (pools, x, out,
 * router weights, logits, codes) starts on a 16-byte boundary, as every
 * cudaMalloc'd or torch-allocated buffer does; a call given another refuses it
 * with FT_ERR_INVALID before any launch. */

/* Create a context on the current CUDA device.
 *   host_layers     host [L] pointers (or NULL): layer l's pool of
 *                   (E + n_shared) blobs at ft_blob_stride() each, in host
 *                   memory that must outlive the context.  Page-locked memory
 *                   is used as is; pageable memory is registered (pinned) here
 *                   and unregistered by ft_destroy.  Resize never reloads it
 *                   ([fa] elastic memory management).
 *   resident_layers host [L] pointers (or NULL): per-layer device copies of
 *                   the same pools; a layer with a non-NULL entry is served
 *                   from it and never touches the cache.  The context
 *                   borrows them: they must outlive it as well.
 *   The library allocates the cache slot arena (CUDA virtual memory, sized by
 *   desc->cache_budget_bytes), device scratch for desc->max_tokens tokens,
 *   a copy stream and events.  Prefill staging buffers (2 layer pools) are
 *   allocated on the first ft_prefetch_layer().
 * Errors: FT_ERR_INVALID (shape limits above, NULL desc/out), FT_ERR_CUDA. */
FT_API ft_status ft_create(const ft_model_desc* desc, const void* const* host_layers,
                    const void* const* resident_layers, ft_ctx** out);

/* Wait for the context's streams, free everything it allocated. */
FT_API ft_status ft_destroy(ft_ctx* ctx);

/* Copy the device status word to the host (synchronising `stream`), clear it,
 * and map it: NaN/+inf logit -> FT_ERR_NONFINITE, bad id -> FT_ERR_INVALID,
 * device wait gave up -> FT_ERR_TIMEOUT; else FT_OK. */
FT_API ft_status ft_sync_status(ft_ctx* ctx, void* stream);

/* ---------------------------------------------------------------------- */
/* hot-path steps (also used by ft_moe_layer_forward)                      */
/* ---------------------------------------------------------------------- */

/* Router logits = x . Wr^T ([hu]: a gate picks 6 of 256 experts per layer).
 *   x dev bf16 [T][H], wr dev fp32 [E][H], logits dev fp32 [T][E].
 * Each bf16*fp32 product is exact in fp64; the sum runs in fp64 in a fixed
 * order (element k joins partial sum (k/4) mod 32 in ascending k; the 32
 * partials meet in an xor butterfly 16,8,4,2,1) and is rounded once to fp32,
 * so results are reproducible bit for bit.  H % 128 == 0. */
FT_API ft_status ft_router_logits(ft_ctx* ctx, const void* x, int64_t T, int32_t H,
                           const float* wr, int32_t E, float* logits, void* stream);

/* Softmax top-k routing ([hu], [no] "Hva er FreeToken?": the router picks a
 * few experts per token).  logits dev fp32 [T][E]; ids dev int32 [T][k] in
 * rank order (logit descending, ties to the lower id, -0 == +0, NaN below
 * -inf); w dev fp32 [T][k]: softmax over all E at the chosen ids, divided by
 * their sum when flags has FT_ROUTE_RENORM.  NaN/+inf logits or a row with no
 * finite logit set the NONFINITE status (ids are still written).  E <= 1024,
 * k <= 16. */
FT_API ft_status ft_moe_route(ft_ctx* ctx, const float* logits, int64_t T, int32_t E, int32_t k,
                       uint32_t flags, int32_t* ids, float* w, void* stream);

/* Permutation of the T*k (token, rank) pairs by expert: histogram, scan and
 * stable scatter.  ids dev int32 [T*k]; offs dev int32 [E+1] (pairs of expert
 * e at positions offs[e]..offs[e+1]-1, ascending token); perm dev int32 [T*k]
 * (perm[pos] = t*k + j); inv dev int32 [T*k] (inv[t*k+j] = pos).  Ids outside
 * [0, E) set the INVALID status and are left out. */
FT_API ft_status ft_moe_permute(ft_ctx* ctx, const int32_t* ids, int64_t T, int32_t k, int32_t E,
                         int32_t* offs, int32_t* perm, int32_t* inv, void* stream);

/* OCP MX quantisation of rows (prefill activations): x dev fp32 [R][K] ->
 * codes dev uint8 [R][K/2] (two e2m1 per byte, element 2i low) and scales dev
 * uint8 laid out in 128x4 atoms over [pad128(R)][K/32] (the blob scale
 * layout).  Block scale = clamp(floor(log2 amax) - 2 + 127, 0, 254), elements
 * rounded to nearest-even onto the e2m1 grid with saturation at 6, sign kept
 * (a negative value that rounds to zero gives code 8).  K % 128 == 0. */
FT_API ft_status ft_quantize_mxfp4(ft_ctx* ctx, const float* x, int64_t R, int32_t K,
                            uint8_t* codes, uint8_t* scales, void* stream);

/* NVFP4 quantisation of rows (the prefill activations of NVFP4 experts;
 * [no] "Hvor raskt kjører modellene?" names the NVFP4 build, the scaling is
 * this library's reading): x dev fp32 [R][K] (finite) -> codes dev uint8
 * [R][K/2] (two e2m1 per byte, element 2i low), scales dev uint8 (E4M3, one
 * per 16 elements) laid out in 128x4 atoms over [pad128(R)][K/16] (the NVFP4
 * blob scale layout), and *tensor_scale (dev fp32) the per-tensor scale s.
 * Every step is one fp32 operation rounded to nearest even:
 *   s = amax / 2688 (amax the largest |x|; s = 0 and every byte 0 when amax is
 *   below 2^-100), g = 1 / (6 s); per block e = E4M3(amax_block * g) (nearest
 *   even, saturating at 448), dq = value(e) * s, r = 1 / dq, codes
 *   e2m1(v * r) (nearest even, saturating at 6, sign kept); dq == 0 gives
 *   codes 0.  A value dequantises to code x value(e) x s.  Uses the
 *   context's one reduction word: calls on one context must not overlap.
 *   K % 128 == 0. */
FT_API ft_status ft_quantize_nvfp4(ft_ctx* ctx, const float* x, int64_t R, int32_t K, uint8_t* codes,
                                   uint8_t* scales, float* tensor_scale, void* stream);

/* ---------------------------------------------------------------------- */
/* layer forward                                                           */
/* ---------------------------------------------------------------------- */

/* One MoE layer on T tokens ([no]: experts fetched to the GPU over PCIe or
 * already cached are computed there, and the partial results are summed
 * exactly):
 *   out[t] = sum_j w[t][j] * FFN_{ids[t][j]}(x[t])  (+ shared FFN(x[t])),
 *   FFN(x) = Wd (silu(Wg x) * (Wu x)), summed over j ascending in fp32,
 *   rounded once to bf16.
 *   x dev bf16 [T][H]; out dev bf16 [T][H] (must not alias x).
 *   router_w dev fp32 [E][H], used when logits_override is NULL.
 *   logits_override dev fp32 [T][E] or NULL.
 *   flags: FT_ACT_BF16 (decode GEMV; T <= 16 and <= max_tokens) or
 *   FT_ACT_MXFP4 / FT_ACT_NVFP4 (prefill grouped GEMM on MXFP4 / NVFP4
 *   weights; any T <= max_tokens), | FT_ROUTE_RENORM.  NVFP4 prefill
 *   quantises x with one per-tensor scale over the T tokens and h with one
 *   over every h row of the layer (routed pairs and the shared expert).
 * Weights come from, in this order: the layer's resident device pool; the
 * prefill staging buffer if ft_prefetch_layer(layer) was issued (the compute
 * stream waits for that copy, [fa] double-buffered prefill); otherwise the
 * expert cache: the selected ids are copied to the host (a stream
 * synchronisation), the global LRU ([no] one LRU across MoE layers; [fa]
 * shared LRU) is updated in ascending expert id, misses are copied from the
 * host pool into their slots on the copy stream, and the experts run once
 * their copies landed.
 * Errors: FT_ERR_INVALID, FT_ERR_NO_SPACE (more distinct experts than
 * slots), FT_ERR_NONFINITE / FT_ERR_TIMEOUT (cache path: checked at its
 * synchronisation), FT_ERR_NOT_FOUND (no pool holds the layer), FT_ERR_CUDA. */
FT_API ft_status ft_moe_layer_forward(ft_ctx* ctx, int32_t layer, const void* x, int64_t T,
                               const float* router_w, const float* logits_override,
                               void* out, uint32_t flags, void* stream);

/* Decode of T tokens (T <= 16) through n_layers consecutive layers, all with
 * resident pools: layer i's output is layer i+1's input.
 *   x dev bf16 [T][H] (input of first_layer), out dev bf16 [T][H] (output of
 *   the last layer; must not alias x); logits dev fp32 [n_layers][T][E]
 *   (router logits of each layer, all ready before the call).
 * Each layer computes what the ft_moe_layer_forward decode path computes, bit
 * for bit.  Because every layer's routing input is known up front, one
 * kernel routes all layers first; then one persistent cooperative kernel runs
 * every layer (waits bounded at 2 s; a timeout sets FT_ERR_TIMEOUT's status
 * bit):
 *   - up to two tokens (when ft_flow_geometry takes the shape): the dataflow
 *     kernel, whose hand-overs between CTAs are tagged words;
 *   - three or four tokens: the same kernel in waves of two tokens (a routing
 *     launch and a dataflow launch per wave; the tokens of a layer do not
 *     interact, so the bits are the same);
 *   - otherwise, or with FT_STACK_COUNTERS: the counter-synchronised kernel
 *     (MXFP4 weights), in which each CTA takes its gate/up and down tiles of
 *     a layer in turn and layers hand over through counters.
 * With FT_STACK_LAYERWISE, or where no persistent kernel takes the shape and
 * format, each layer runs as a gate/up and a down kernel instead.
 * Intermediate activations live in context scratch; calls on different
 * streams must not overlap.
 * flags: FT_ROUTE_RENORM | FT_STACK_LAYERWISE | FT_STACK_COUNTERS.
 * Errors: FT_ERR_INVALID, FT_ERR_STATE (a layer is not resident), FT_ERR_CUDA. */
FT_API ft_status ft_moe_stack_forward(ft_ctx* ctx, int32_t first_layer, int32_t n_layers, const void* x, int64_t T,
                                      const float* logits, void* out, uint32_t flags, void* stream);

/* Copy the ids [T][k] and weights [T][k] of the last decode or prefill
 * routing (n = T*k entries) to ids / w (device or host memory), on `stream`. */
FT_API ft_status ft_last_routing(ft_ctx* ctx, int32_t* ids, float* w, int64_t n, void* stream);

/* ---------------------------------------------------------------------- */
/* expert cache ([no] global LRU; [fa] elastic resize)                     */
/* ---------------------------------------------------------------------- */

/* Slot of (layer, expert), touching it as most recent; *slot = -1 on a miss
 * (no other change).  FT_ERR_INVALID on bad ids or no cache. */
FT_API ft_status ft_expert_cache_lookup(ft_ctx* ctx, int32_t layer, int32_t expert, int32_t* slot);

/* Make (layer, expert) resident: a hit only touches it; a miss evicts the
 * least-recent key when full, then copies the blob from the host pool into
 * its slot on the copy stream (`stream` waits for that copy).  *slot gets the
 * slot, *evicted_key the evicted layer*E+expert or -1.  FT_ERR_NO_SPACE if
 * the capacity is 0. */
FT_API ft_status ft_expert_cache_insert(ft_ctx* ctx, int32_t layer, int32_t expert, int32_t* slot,
                                 int64_t* evicted_key, void* stream);

/* Change the cache budget ([fa]: resize without restart or pool reload).
 * Waits for the context's streams.  Shrink: evict least-recent keys until the
 * survivors fit, move survivors from slots >= the new capacity to the lowest
 * free slots below it (device-to-device copies), then unmap the physical
 * memory past the new size.  Grow: map more physical memory.  The host pool is
 * not touched.  FT_ERR_INVALID for a negative budget; FT_ERR_CUDA if physical
 * memory cannot be mapped. */
FT_API ft_status ft_expert_cache_resize(ft_ctx* ctx, int64_t new_budget_bytes);

/* Decode-time next-layer prefetch ([ro] predictive preloading of the
 * experts the coming tokens will likely use; [fa] adjacent tokens' expert
 * paths overlap).  With per_layer > 0 (at most 16), after each cache step at
 * layer l the context counts that step's experts, then copies up to per_layer
 * experts of layer (l + 1) mod n_layers into the cache: those selected at
 * least once so far, most often first (ties to the lower id), skipping
 * resident ones.  Each is inserted as most recent (a FT_EV_PREFETCH event),
 * evicting when full the least recent key that is neither in the step's set
 * nor of layer l + 1.  The copies run on the copy stream behind the step's
 * own misses; an expert hit before its prefetch copy landed waits for that
 * copy.  0 turns it off (the default).  FT_ERR_INVALID outside [0, 16] or
 * without a cache. */
FT_API ft_status ft_cache_prefetch(ft_ctx* ctx, int32_t per_layer);

/* Copy out the cache events recorded since the last call (HIT, MISS, EVICT,
 * MOVE in order) and clear them.  *n = events written (<= cap); if more were
 * recorded than cap the rest are dropped and FT_ERR_NO_SPACE is returned.
 * Between two calls the context keeps at most 4,194,304 events (80 MiB); the
 * events after that are not recorded, and the next call copies out the ones
 * kept and returns FT_ERR_NO_SPACE. */
FT_API ft_status ft_cache_trace(ft_ctx* ctx, ft_cache_event* buf, int64_t cap, int64_t* n);

/* Counters since creation (or the last reset). */
FT_API ft_status ft_cache_stats_get(ft_ctx* ctx, ft_cache_stats* out, int32_t reset);

/* ---------------------------------------------------------------------- */
/* prefill prefetch ([fa]: next layer's experts cross PCIe while the GPU  */
/* computes the current one; [no]: streams the next layer pack)            */
/* ---------------------------------------------------------------------- */

/* Start copying layer `layer`'s whole pool from host into staging buffer
 * (layer & 1) on the copy stream.  The copy first waits until the last
 * forward that read that buffer (recorded on its compute stream) finished.
 * Returns at once.  FT_ERR_NOT_FOUND without a host pool; FT_ERR_CUDA. */
FT_API ft_status ft_prefetch_layer(ft_ctx* ctx, int32_t layer, void* compute_stream);

/* ---------------------------------------------------------------------- */
/* parity export                                                           */
/* ---------------------------------------------------------------------- */

/* Dequantise matrix `mat` (0 = Wg, 1 = Wu, 2 = Wd) of a blob at dev pointer
 * `blob` to fp32 out dev [rows][K]: code value x UE8M0 scale, exact in fp32
 * unless the product overflows (then +-inf) ([no] "MXFP4": e2m1 values with
 * per-32 power-of-two scales).  The rows pass through the decode kernels' own
 * tile: staged into shared memory as the decode GEMVs stage them, read back
 * chunk by chunk and converted by the same e2m1 -> f16 decoder their dot
 * products use.  FT_ERR_INVALID for a shape the decode kernels do not take. */
FT_API ft_status ft_debug_dequant(ft_ctx* ctx, const void* blob, int32_t mat, float* out, void* stream);

/* Tile geometry the decode kernels use for hidden H and intermediate I
 * (host only, no device needed).  out[0..9] describe the gate/up tile and
 * out[10..19] the down tile, each: K, 32-code chunks of K, lanes per row group
 * (lpr), row groups per warp (rpw), K parts, row sets, lane groups per CTA, R
 * rows per tile, shared-memory bytes of a per-layer CTA, 1 if the tile is
 * taken; out[20] threads per CTA, out[21] the shared-memory limit of a tile,
 * out[22] 1 if the persistent kernel takes a stack of n_layers layers of this
 * shape, out[23] its counter words per layer.  FT_ERR_INVALID on a bad shape. */
FT_API ft_status ft_decode_geometry(int32_t hidden, int32_t inter, int32_t n_layers, int64_t out[24]);

/* Geometry of the dataflow decode kernel that ft_moe_stack_forward runs for
 * one or two tokens, and in waves of two for three or four (host only, no
 * device needed; T is the tokens of one launch): out[0] = 1 if it takes
 * this shape, batch T, stack depth and weight format (else the
 * counter-synchronised or the per-layer kernels run), out[1] = rows of a down tile over all units,
 * out[2] = shared memory of a CTA in bytes.  FT_ERR_INVALID on a bad shape. */
FT_API ft_status ft_flow_geometry(int32_t hidden, int32_t inter, int32_t T, int32_t top_k, int32_t n_shared,
                                  int32_t n_experts, int32_t n_layers, int32_t weight_format, int64_t out[3]);

/* Failure injection for tests: none of these fault or hang a GPU.
 *
 * ft_debug_device_wait: launch, on `stream`, one CTA that waits for a device
 * flag nothing ever sets, with the bounded wait the persistent decode kernel
 * uses between layers, limited to timeout_us microseconds (1 .. 2,000,000);
 * when the limit runs out the CTA sets the timeout bit of the context's
 * status word and returns, so the next ft_sync_status reports
 * FT_ERR_TIMEOUT and the context stays usable.  Errors: FT_ERR_INVALID,
 * FT_ERR_CUDA.
 *
 * ft_debug_host_wait_limit: the limit (seconds, > 0) of the context's bounded
 * host waits on device events (the cache path's wait for the routed ids
 * before its LRU step); the default is 30 s.  A wait that runs out returns
 * FT_ERR_TIMEOUT with the cache unchanged; the work already queued stays
 * queued.
 *
 * ft_debug_fail_copy: the n-th host-to-device expert copy the cache issues
 * from now on (n >= 1; 0 turns injection off) fails instead of being issued:
 * the call returns FT_ERR_CUDA, the key whose copy failed is dropped from the
 * cache again (a MISS then an EVICT event in the trace), keys fetched earlier
 * in the same step stay resident, and a retry of the step fetches the dropped
 * key. */
FT_API ft_status ft_debug_device_wait(ft_ctx* ctx, int64_t timeout_us, void* stream);

/* Test hook for the persistent decode kernel's tagged hand-over words.  Each
 * such word carries a 32-bit tag (launch counter << 7 | layer) that repeats
 * every 2^25 launches; the routing kernel zeroes all tagged words when the
 * counter wraps, so that a word left from 2^25 launches earlier cannot pass
 * for one of the current launch.  This call waits for the device, sets the
 * launch counter to `epoch` and, when poison_layer is in [0, 127], fills every
 * tagged word with a NaN carrying the tag the next launch gives layer
 * poison_layer (a stale word of exactly the kind the zeroing removes).
 * Errors: FT_ERR_INVALID, FT_ERR_STATE (no persistent kernel in this
 * context), FT_ERR_CUDA. */
FT_API ft_status ft_debug_stack_epoch(ft_ctx* ctx, uint32_t epoch, int32_t poison_layer);

/* Phase timeline of the dataflow stack kernel, for profiling: with buf (dev
 * uint64 [n_words]) attached, each later ft_moe_stack_forward that runs the
 * dataflow kernel over n layers with at least n * (number of SMs) * 8 words
 * writes, at [layer][CTA][0..7], the %globaltimer nanoseconds at which the
 * CTA began the layer [0], had its first gate/up tile's input and weights
 * [1], had that tile's dot products [7], had published its h [2], had its
 * first down tile's h and weights [3], had that tile's dot products [5],
 * had stored its combined rows [6] and had left the down phase [4] (0 where
 * the CTA had no tile of that phase).  NULL detaches it.  The kernel's
 * results do not change. */
FT_API ft_status ft_debug_stack_timeline(ft_ctx* ctx, uint64_t* buf, int64_t n_words);
FT_API ft_status ft_debug_host_wait_limit(ft_ctx* ctx, double seconds);
FT_API ft_status ft_debug_fail_copy(ft_ctx* ctx, int64_t n);

/* ---------------------------------------------------------------------- */
/* measurement                                                             */
/* ---------------------------------------------------------------------- */

/* FP4 tensor-core peak probe: one CTA per SM issues iters (1 .. 65536)
 * rounds of four tcgen05.mma kind::mxf4 (M = N = 128, K = 64, MXFP4 x MXFP4
 * with UE8M0 block scales, the prefill GEMM's instruction) on operands held
 * in shared memory, into a tensor-memory accumulator, on `stream`.  It
 * performs (*grid) * iters * 4 * 2 * 128 * 128 * 64 floating-point operations
 * and reads no global memory while it runs, so the launch time measures the
 * tensor pipe.  sink: dev fp32 [number of SMs], one accumulator value per CTA;
 * status: dev int32, bit 4 set if the wait for the tensor pipe gave up
 * (200 ms).  *grid = CTAs launched.  Errors: FT_ERR_INVALID, FT_ERR_CUDA. */
FT_API ft_status ft_fp4_mma_probe(int64_t iters, float* sink, int32_t* status, int32_t* grid, void* stream);

/* Kernel classes of the per-kernel timers. */
#define FT_K_ROUTER_LOGITS 0
#define FT_K_TOPK          1
#define FT_K_PERMUTE       2
#define FT_K_GATE_UP       3   /* decode gate/up + SwiGLU GEMV */
#define FT_K_DOWN_COMBINE  4   /* decode down GEMV + combine */
#define FT_K_QUANT_X       5   /* prefill activation quantiser */
#define FT_K_GEMM_GATE_UP  6   /* prefill grouped GEMM, gate/up + SwiGLU + quantise h */
#define FT_K_GEMM_DOWN     7   /* prefill grouped GEMM, down */
#define FT_K_COMBINE       8   /* prefill combine */
#define FT_K_DEC_STACK     9   /* persistent decode kernel over a stack of layers */
#define FT_K_QUANT_H       10  /* NVFP4 prefill: quantiser of h (after the gate/up GEMM) */
#define FT_K_COUNT         11

/* Turn per-kernel CUDA-event timing on (1) or off (0).  While on, every
 * kernel launch of the forward path is bracketed by events on its stream (and
 * consecutive layers are not overlapped).  Launches made under stream capture
 * record their events into the graph: each ft_kernel_timing_read after a
 * replay adds that replay's times.  Enabling or disabling resets the counters
 * and releases the events, so destroy graphs that hold them first. */
FT_API ft_status ft_kernel_timing_enable(ft_ctx* ctx, int32_t on);

/* Synchronise, then fill ms[i] (total device time) and launches[i] for the
 * first n kernel classes (FT_K_*) accumulated since timing was enabled. */
FT_API ft_status ft_kernel_timing_read(ft_ctx* ctx, double* ms, int64_t* launches, int32_t n);

/* ---------------------------------------------------------------------- */
/* forward without allocation                                              */
/* ---------------------------------------------------------------------- */

/* Largest scratch one ft_moe_layer_forward_noalloc call may use (bytes). */
#define FT_NOALLOC_SCRATCH_BYTES (8u << 20)

/* The decode forward of ft_moe_layer_forward for callers that cannot
 * allocate device memory: processes whose device memory belongs entirely to
 * another allocator, and latency-critical paths that cannot afford the device
 * synchronisation cudaMalloc / cudaFree may bring.  The write-ups describe no
 * counterpart; this is a library convenience.
 *
 * Needs no context and allocates nothing: its scratch is one static device
 * array of FT_NOALLOC_SCRATCH_BYTES that every GPU loading the library keeps
 * until the process exits.  The first call on a device looks up that array's
 * device address (cudaGetSymbolAddress) with the device current; make that
 * first call before any stream capture on the device.  All calls share the
 * array and it keeps the last call's contents: calls whose work overlaps on
 * the GPU (other streams, other host threads) race and corrupt each other, so
 * order them on one stream.
 *   shape       hidden, inter (multiples of 128), n_experts (<= 1024), top_k
 *               (<= 16), n_shared (0 or 1), as in ft_model_desc
 *   layer_pool  dev: the layer's (n_experts + n_shared) blobs at
 *               ft_blob_stride(hidden, inter) each, resident on the device
 *   x, out      dev bf16 [T][hidden], T in [0, 16]; out must not alias x
 *   router_w / logits_override, flags   as in ft_moe_layer_forward
 *               (FT_ACT_MXFP4 is rejected: decode path only)
 *   status      dev int32 or NULL: device-detected errors (bits: 1 NaN/+inf
 *               logit, 2 bad id) are OR-ed into it; the caller clears it.
 *               With NULL they are dropped.
 * Errors: FT_ERR_INVALID for bad arguments or when the call's scratch
 * (routing arrays plus (T*top_k + n_shared*T) * inter * 4 bytes of
 * activations) exceeds FT_NOALLOC_SCRATCH_BYTES; FT_ERR_CUDA. */
FT_API ft_status ft_moe_layer_forward_noalloc(int32_t hidden, int32_t inter, int32_t n_experts, int32_t top_k,
                                              int32_t n_shared, const void* layer_pool, const void* x, int64_t T,
                                              const float* router_w, const float* logits_override, void* out,
                                              uint32_t flags, int32_t* status, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FT_MOE_H */

// Small-batch decode kernels: a routing kernel that writes one compact routing
// record per layer, then either one persistent kernel for a stack of layers or,
// per layer, a gate/up + SwiGLU GEMV and a down GEMV with the combine (FP4
// tiles staged in shared memory; each lane owns a 32-code chunk of K).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "ft_common.cuh"

namespace ft {

constexpr int kMaxPairs = 256;  // T * k
constexpr int kMaxUnits = 257;  // distinct experts + shared

// Routing of one layer for T <= 16 tokens (device memory, written by k_route).
struct alignas(16) Route {
  int32_t ids[kMaxPairs];    // [t*k + j], rank order
  float w[kMaxPairs];        // combine weights
  int32_t pos[kMaxPairs];    // permuted position of pair f (= inv)
  int32_t perm[kMaxPairs];   // pair at permuted position
  int32_t unit_e[kMaxUnits]; // distinct experts, ascending
  int32_t unit_p0[kMaxUnits];
  int32_t unit_m[kMaxUnits];
  uint8_t first[kMaxPairs];  // pair is its expert's lowest-token pair
  int32_t n_active;
  int32_t bad;
  int32_t pad[2];
};

struct RouteArgs {
  const float* logits;  // fp32 [n_layers][T][E], layers layer_stride floats apart
  int64_t layer_stride; // 0: T * E
  int T, E, k, renorm, n_layers;
  Route* rec;           // [n_layers]
  int32_t* ids_out;     // [T*k] of the last layer, or NULL
  float* w_out;
  int* status;
  int* sync;            // [n_layers][sync_stride] zeroed by CTA l for layer l, or NULL
  int sync_stride;
  uint32_t* epoch;      // launch counter the persistent kernel tags its h with; CTA 0 adds 1, or NULL
  uint64_t* tagged;     // the persistent kernel's tagged words: CTA 0 zeroes them when the counter wraps
  int64_t tagged_words;
};

// Launch counter after `e`: e + 1, skipping values whose tags (e << 7 | layer,
// 32 bits) could equal a zeroed word's.  *wrapped is set when it skipped, i.e.
// when the tags start repeating those of 2^25 launches before.
__host__ __device__ inline uint32_t next_epoch(uint32_t e, bool* wrapped) {
  uint32_t n = e + 1u;
  const bool w = (n << 7) == 0u;
  if (w) n += 1u;
  if (wrapped) *wrapped = w;
  return n;
}

struct DecodeArgs {
  const uint16_t* x;       // bf16 [T][H]
  const Route* rec;        // this layer's routing record
  int T, H, I, E, k, n_shared;
  int max_units;           // routed unit slots: min(E, T*k)
  const uint8_t* const* eptr;  // [E + n_shared] blob pointers
  BlobLayout lay;
  float* h;                // [T*k + n_shared*T][I]
  float* y;                // [T*k + n_shared*T][H]
  uint16_t* out;           // bf16 [T][H]
  int* counters;           // [H/8] combine counters, zero before the first launch
  int* status;
  // Units this launch takes: all (n_sel == 0), or the units sel[0 .. n_sel).
  // The cache path runs the resident experts at once and each fetched expert
  // after its own copy; the last down CTA of a row block, over all launches of
  // the layer, does the combine.
  int n_sel;
  uint16_t sel[kMaxUnits];
};

// True when the decode kernels take this shape in weight format fmt (hidden
// and inter multiples of 128, both at most 16384).
bool decode_supported(int H, int I, int fmt = kFmtMx);
// Tile geometry of the decode kernels for hidden H and intermediate I:
// out[0..9] gate/up tile, out[10..19] down tile, each K, chunks, lpr, rpw,
// parts, rsets, groups, R, shared bytes of a per-layer CTA, taken (0/1);
// out[20] threads per CTA, out[21] the shared-memory limit of a tile.
void decode_geometry(int H, int I, int64_t* out);
cudaError_t launch_route(const RouteArgs& a, cudaStream_t s);
// Matrix mat (0 Wg, 1 Wu, 2 Wd) of one blob dequantised to fp32 [rows][K]
// through the GEMV tile's staging and code decoder (shape must satisfy
// decode_supported).
cudaError_t launch_dec_dequant(const uint8_t* blob, const BlobLayout& lay, int mat, int H, int I, float* out,
                               cudaStream_t s);
// pdl: launch as a programmatic dependent of the previous kernel in the
// stream.  The gate/up kernel reads its routing record and pointer table
// before griddepcontrol.wait, so it may only be launched that way when both
// were complete before the previous kernel started; the down kernel reads
// nothing produced by gate/up before its wait.
cudaError_t launch_dec_gate_up(const DecodeArgs& a, bool pdl, cudaStream_t s);
cudaError_t launch_dec_down(const DecodeArgs& a, bool pdl, cudaStream_t s);

// Persistent decode over n_layers consecutive layers in one cooperative launch.
struct StackArgs {
  const uint16_t* x0;      // bf16 [T][H] input of the first layer
  uint16_t* out;           // bf16 [T][H] output of the last layer
  uint16_t* xbuf[2];       // bf16 [T][H] ping-pong between layers
  const Route* rec;        // [n_layers] routing records
  const uint8_t* const* eptr;  // [n_layers][n_blobs] blob pointers
  int n_layers, n_blobs;
  int T, H, I, E, k, n_shared;
  BlobLayout lay;
  float* h;                // [T*k + n_shared*T][I]
  float* y;                // [T*k + n_shared*T][H]
  int* sync;               // [n_layers][sync_stride], zero at launch
  int sync_stride;         // >= stack_sync_stride(H, I)
  int* status;
};

// True when the persistent kernel takes this shape and stack depth (both
// tiles of a layer and the per-layer tile table fit in shared memory).
bool stack_supported(int H, int I, int n_layers);
int stack_sync_stride(int H, int I);
cudaError_t launch_dec_stack(const StackArgs& a, cudaStream_t s);

// Dataflow decode over n_layers consecutive layers for one or two tokens
// (ft_decode_flow.cu): one cooperative launch, one CTA per SM; h and the next
// layer's x travel as tagged words, the down tiles span every unit and
// combine their rows themselves.
struct FlowArgs {
  const uint16_t* x0;          // bf16 [T][H] input of the first layer
  uint16_t* out;               // bf16 [T][H] output of the last layer
  const Route* rec;            // [n_layers] routing records
  const uint8_t* const* eptr;  // [n_layers][n_blobs] blob pointers
  int n_layers, n_blobs;
  int T, H, I, E, k, n_shared;
  BlobLayout lay;
  uint64_t* h_tagged;          // [T*k + n_shared*T][I] words: tag << 32 | fp32
  uint64_t* x_tagged;          // [T][H/2] words: tag << 32 | two bf16
  const uint32_t* epoch;       // advanced by the routing kernel before this launch
  int rows_cap;                // down-tile rows over all units (flow_geometry)
  int* status;
  // NULL, or [n_layers][gridDim][8] %globaltimer stamps of each CTA: gate/up
  // start, x staged, h published, down h staged, x published (0 where the CTA
  // had no tile of the phase)
  uint64_t* timeline;
};
struct FlowGeom {
  int rows_cap;
  size_t smem;
  bool ok;                     // the dataflow kernel takes this shape, batch and depth
};
FlowGeom flow_geometry(int H, int I, int T, int k, int S, int E, int n_layers, int fmt = kFmtMx);
cudaError_t launch_dec_flow(const FlowArgs& a, cudaStream_t s);

// One CTA waiting, with the persistent kernel's bounded wait, for *flag >= 1;
// sets the timeout bit of *status after limit_ns.
cudaError_t launch_debug_wait(const int* flag, int* status, uint64_t limit_ns, cudaStream_t s);

}  // namespace ft

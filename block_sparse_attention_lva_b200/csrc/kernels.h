// kernels.h -- host-side launchers implemented by the kernel translation units.
// Arguments are validated by the C ABI layer (api.cu) before these are called; each
// launcher returns the cudaError_t of its launch(es).
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "lva.h"

namespace lva {

// Per-device setup done once (a kernel's shared-memory limit, a looked-up attribute).  The
// flags are atomic so that concurrent host threads are safe; the setup itself must be
// idempotent, since two threads may both run it before either sets the flag.  Devices past
// the cache run the setup on every call.
constexpr int kMaxCachedDevices = 64;
using DeviceFlags = std::atomic<bool>[kMaxCachedDevices];

template <class F>
cudaError_t once_per_device(DeviceFlags& done, F&& setup) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < kMaxCachedDevices;
  if (cached && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = setup();
  if (e == cudaSuccess && cached) done[dev].store(true, std::memory_order_release);
  return e;
}

// Streaming multiprocessors of the current device (looked up once per device; 148 if the
// query fails).
inline int sm_count() {
  static std::atomic<int> cached[kMaxCachedDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  const bool cacheable = dev >= 0 && dev < kMaxCachedDevices;
  if (cacheable) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (cacheable) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

struct ReorderArgs {
  const void* src;
  void* dst;
  int64_t planes;
  int T, H, W, tt, th, tw;
  int64_t n_valid, n_pad;
  int64_t row_bytes;
  int inverse;
};
cudaError_t launch_reorder(const ReorderArgs& a, cudaStream_t stream);

struct MaskArgs {
  int kind;
  int mask_heads;
  int block_size;
  int64_t n_pad, n_valid;
  int64_t unit_tokens;
  int radius, num_anchors, step, group_blocks, budget_frames;
  const uint8_t* dense;
  int32_t* row_ptr;
  int32_t* col_idx;
  int32_t* nnz_out;
};
cudaError_t launch_build_mask(const MaskArgs& a, cudaStream_t stream);

// Workspace bytes of the packed static-mask build (0 for the other kinds), and the build
// itself: the dense mask is read once into bits (workspace), the counts are scanned by
// several CTAs when there are many rows, and the bits are expanded into the CSR.
int64_t mask_workspace_bytes(int kind, int64_t rows, int64_t nb);
cudaError_t launch_build_mask_packed(const MaskArgs& a, void* workspace, cudaStream_t stream);

// The packed build with its workspace in the library's own static device array (at most
// mask_noalloc_scratch_bytes(); the caller checks the size first).
int64_t mask_noalloc_scratch_bytes();
cudaError_t launch_build_mask_noalloc(const MaskArgs& a, cudaStream_t stream);

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int B, H;
  int64_t n_pad, n_valid;
  int d, block_size;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int64_t col_len;
  int mask_heads;
  float scale;
  const int32_t* query_src;  // NULL or [src_heads, nb]
  int src_heads;
  int* err;  // device error word
  void* o_raster;            // NULL, or O in raster order [B, H, n_valid, d] instead of o
  int T, Hg, Wg, tt, th, tw; // latent grid and tile (used with o_raster)
  int gather_windows;        // 0, or m: q, k, v are read window-transposed (see api.cu)
  int gather_window;         // w, the tokens per window, with gather_windows
  int lse_only;              // 1: only LSE is computed (v, o and o_raster unused)
};
cudaError_t launch_attn(const AttnArgs& a, cudaStream_t stream, const char** why);

struct BroadcastArgs {
  void* o;
  float* lse;
  int B, H;
  int64_t n_pad;
  int d, block_size;
  const int32_t* query_src;
  int src_heads;
  int* err;
};
cudaError_t launch_broadcast(const BroadcastArgs& a, cudaStream_t stream);

struct EnergyArgs {
  const void* q;
  const void* k;
  const float* lse;
  float* energy;
  int B, H;
  int64_t n_pad, n_valid;
  int d, block_size;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int64_t col_len;
  int mask_heads;
  float scale;
  int* err;
};
cudaError_t launch_energy(const EnergyArgs& a, cudaStream_t stream, const char** why);

struct SelectArgs {
  const float* energy;   // [rows, nb]
  uint8_t* mask;         // [rows, nb]
  int64_t rows;
  int nb;
  double eps;
  int* err;
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream);

struct AggregateArgs {
  const uint8_t* masks;  // [prompts, count]
  uint8_t* out;          // [count]
  int prompts;
  int64_t count;
  double threshold;      // rho * prompts, in float64
};
cudaError_t launch_aggregate(const AggregateArgs& a, cudaStream_t stream);

// Largest nb the selection supports (its sort holds a row in shared memory).
constexpr int kSelectMaxBlocks = 4096;

// 2D tensor map over a bf16 [rows, d] row-major matrix, box of 64 elements x box_rows,
// 128-byte swizzle (from tmap.cu).  Returns false when the driver entry point is missing
// or the encoding fails.
bool make_rows_map(CUtensorMap* m, const void* base, int64_t rows, int d, int box_rows);

// 3D tensor map over a bf16 [planes * windows, window, d] buffer, box of 64 elements x 1
// position x box_rows windows: one box gathers the rows of box_rows consecutive windows at
// one position, i.e. box_rows consecutive rows of the window-transposed order.
bool make_window_gather_map(CUtensorMap* m, const void* base, int64_t planes, int windows, int window,
                            int d, int box_rows);

// Device error word of the current device (from api.cu).
int* device_error_word();

// Sets the calling thread's lva_last_error_message (printf-style) and returns `status`
// (from api.cu; an empty message for LVA_OK).
lva_status set_error_message(lva_status status, const char* fmt, ...);

// Bounded-wait self-test (selftest.cu): mode 0 = nothing arrives, 1 = abort flag raised,
// 2 = the peer arrives.
cudaError_t launch_wait_selftest(int mode, int* err, cudaStream_t stream);

}  // namespace lva

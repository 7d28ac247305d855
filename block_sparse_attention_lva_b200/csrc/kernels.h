// kernels.h -- host-side launchers implemented by the kernel translation units.
// Arguments are validated by the C ABI layer (api.cu) before these are called; each
// launcher returns the cudaError_t of its launch(es).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace lva {

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

// Device error word of the current device (from api.cu).
int* device_error_word();

}  // namespace lva

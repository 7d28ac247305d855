// layer.cu -- one attention layer from and to pinned host memory, with the copies overlapped.
//
// lva_layer_step_host chains the library's own calls for one layer of a video diffusion
// transformer -- the tile reorder of Q, K and V, the CSR of the step's block mask, the
// block-sparse attention with the inverse reorder fused into its epilogue -- per group of
// heads, with each group's host-to-device copy on one stream, its compute on another and its
// device-to-host copy on a third, ordered by caller-created events.  So group g + 1 is copied
// in while group g is computed and group g - 1 is copied out, and two buffer sets used
// alternately let consecutive steps overlap too.  Nothing is allocated here.
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"
#include "lva.h"

namespace lva {
namespace {

bool is_pinned_host(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();   // an unregistered pointer may set the sticky-free last error
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

}  // namespace

// Argument checks of lva_layer_step_host that need no device.
lva_status check_layer_step(const void* qkv_host, const void* o_host, const float* lse_host,
                            const lva_layer_shape* sh, const lva_mask_params* mask,
                            const lva_host_step_buffers* bufs, int head_groups, int build_mask,
                            const int32_t* query_src, int src_heads, int* groups_out, int* heads_out,
                            const char** why) {
  *why = "";
  if (sh == nullptr || mask == nullptr || bufs == nullptr) { *why = "null shape, mask or buffers"; return LVA_ERR_INVALID_ARG; }
  if (sh->B < 1 || sh->H < 1) { *why = "need B >= 1 and H >= 1"; return LVA_ERR_INVALID_ARG; }
  if (sh->d != 64 && sh->d != 128) { *why = "head dim must be 64 or 128"; return LVA_ERR_UNSUPPORTED; }
  if (sh->block_size != 64 && sh->block_size != 128) { *why = "block_size must be 64 or 128"; return LVA_ERR_UNSUPPORTED; }
  if (!(sh->scale == sh->scale)) { *why = "scale is NaN"; return LVA_ERR_INVALID_ARG; }
  if (sh->T < 1 || sh->Hg < 1 || sh->Wg < 1 || sh->tile_t < 1 || sh->tile_h < 1 || sh->tile_w < 1) {
    *why = "grid and tile extents must be >= 1"; return LVA_ERR_INVALID_ARG;
  }
  const int64_t n = int64_t(sh->T) * sh->Hg * sh->Wg;
  if (mask->block_size != sh->block_size || mask->n_valid != n || mask->n_pad < n ||
      mask->n_pad % sh->block_size != 0 || mask->n_pad - n >= sh->block_size) {
    *why = "mask n_valid / n_pad / block_size must be the grid's (n_pad = N rounded up to a block)";
    return LVA_ERR_INVALID_ARG;
  }
  if (mask->mask_heads != 1 && mask->mask_heads != sh->H) { *why = "mask_heads must be 1 or H"; return LVA_ERR_INVALID_ARG; }
  const int64_t max_nnz = lva_block_mask_max_nnz(mask);
  if (max_nnz <= 0) { *why = "invalid mask parameters"; return LVA_ERR_INVALID_ARG; }
  if (int64_t(sh->B) * sh->H * mask->n_pad >= (int64_t(1) << 31)) { *why = "B*H*n_pad must be < 2^31"; return LVA_ERR_UNSUPPORTED; }
  if (head_groups < 1) { *why = "head_groups must be >= 1"; return LVA_ERR_INVALID_ARG; }
  if (qkv_host == nullptr || o_host == nullptr || lse_host == nullptr) { *why = "null host buffer"; return LVA_ERR_INVALID_ARG; }
  if (bufs->qkv_stage == nullptr || bufs->o_stage == nullptr || bufs->lse_stage == nullptr ||
      bufs->qkv_tile == nullptr || bufs->row_ptr == nullptr || bufs->col_idx == nullptr || bufs->nnz == nullptr ||
      bufs->events == nullptr) {
    *why = "null device buffer or event array"; return LVA_ERR_INVALID_ARG;
  }
  if (query_src != nullptr && bufs->o_tile == nullptr) { *why = "repetitive heads need o_tile"; return LVA_ERR_INVALID_ARG; }
  if (query_src != nullptr && src_heads != 1 && src_heads != sh->H) { *why = "src_heads must be 1 or H"; return LVA_ERR_INVALID_ARG; }
  if (bufs->col_len < 0 || bufs->col_len > bufs->col_capacity) { *why = "need 0 <= col_len <= col_capacity"; return LVA_ERR_INVALID_ARG; }
  if (build_mask && bufs->col_capacity < max_nnz) { *why = "col_capacity below lva_block_mask_max_nnz"; return LVA_ERR_CAPACITY; }
  // Groups: up to ceil(head_groups / B) per batch element, each a run of `heads` heads.
  const int want = (head_groups + sh->B - 1) / sh->B;
  const int per_b_max = want < sh->H ? want : sh->H;
  const int heads = (sh->H + per_b_max - 1) / per_b_max;
  const int groups = sh->B * ((sh->H + heads - 1) / heads);
  if (bufs->num_events < 2 * groups + 2) { *why = "too few events (need 2 * groups + 2)"; return LVA_ERR_INVALID_ARG; }
  *groups_out = groups;
  *heads_out = heads;
  return LVA_OK;
}

}  // namespace lva

using namespace lva;

extern "C" lva_status lva_layer_step_host(const void* qkv_host, void* o_host, float* lse_host,
                                          const lva_layer_shape* sh, const lva_mask_params* mask,
                                          const uint8_t* dense_mask, int build_mask, const int32_t* query_src,
                                          int src_heads, const lva_host_step_buffers* bufs, int head_groups,
                                          cudaStream_t compute, cudaStream_t h2d, cudaStream_t d2h,
                                          cudaEvent_t* done) {
  int groups = 0, heads = 0;
  const char* why = "";
  lva_status st = check_layer_step(qkv_host, o_host, lse_host, sh, mask, bufs, head_groups, build_mask, query_src,
                                   src_heads, &groups, &heads, &why);
  if (st != LVA_OK) return set_error_message(st, "layer_step_host: %s", why);
  if (!is_pinned_host(qkv_host) || !is_pinned_host(o_host) || !is_pinned_host(lse_host))
    return set_error_message(LVA_ERR_INVALID_ARG, "layer_step_host: host buffers must be pinned (page-locked) memory");
  const int B = sh->B, H = sh->H, d = sh->d, bs = sh->block_size;
  const int64_t N = mask->n_valid, n_pad = mask->n_pad, nb = n_pad / bs;
  const int per_b = groups / B;
  const size_t row = size_t(d) * 2;                                   // bf16 row bytes
  const size_t plane_in = size_t(N) * row, plane_tile = size_t(n_pad) * row;
  const size_t tensor_in = size_t(B) * H * plane_in, tensor_tile = size_t(B) * H * plane_tile;
  cudaEvent_t* ev = bufs->events;
  cudaEvent_t staging_free = ev[2 * groups], out_free = ev[2 * groups + 1];
  auto cuda = [](cudaError_t e, const char* what) -> lva_status {
    if (e == cudaSuccess) return LVA_OK;
    return set_error_message(LVA_ERR_CUDA, "layer_step_host: %s: %s", what, cudaGetErrorString(e));
  };
#define LVA_TRY(x) do { lva_status s_ = (x); if (s_ != LVA_OK) return s_; } while (0)

  // --- host to device, per group: this buffer set's staging was last read by its previous
  // step's reorders (never-recorded events complete at once)
  LVA_TRY(cuda(cudaStreamWaitEvent(h2d, staging_free, 0), "wait staging"));
  const char* qkv_h = static_cast<const char*>(qkv_host);
  char* stage = static_cast<char*>(bufs->qkv_stage);
  for (int g = 0; g < groups; ++g) {
    const int b = g / per_b, h0 = (g % per_b) * heads, h1 = h0 + heads < H ? h0 + heads : H;
    if (h0 >= H) { LVA_TRY(cuda(cudaEventRecord(ev[g], h2d), "record")); continue; }
    for (int t = 0; t < 3; ++t) {
      const size_t off = size_t(t) * tensor_in + (size_t(b) * H + h0) * plane_in;
      LVA_TRY(cuda(cudaMemcpyAsync(stage + off, qkv_h + off, size_t(h1 - h0) * plane_in, cudaMemcpyHostToDevice, h2d),
                   "copy in"));
    }
    LVA_TRY(cuda(cudaEventRecord(ev[g], h2d), "record"));
  }

  // --- compute: outputs of this buffer set were last read by its previous step's copies out
  LVA_TRY(cuda(cudaStreamWaitEvent(compute, out_free, 0), "wait outputs"));
  if (build_mask) {
    LVA_TRY(lva_build_block_mask(mask, dense_mask, bufs->row_ptr, bufs->col_idx, bufs->col_capacity, bufs->nnz,
                                 compute));
  }
  char* tile = static_cast<char*>(bufs->qkv_tile);
  char* o_st = static_cast<char*>(bufs->o_stage);
  for (int g = 0; g < groups; ++g) {
    const int b = g / per_b, h0 = (g % per_b) * heads, h1 = h0 + heads < H ? h0 + heads : H;
    if (h0 < H) {
      const int hn = h1 - h0;
      const size_t p0 = size_t(b) * H + h0;
      LVA_TRY(cuda(cudaStreamWaitEvent(compute, ev[g], 0), "wait copy in"));
      for (int t = 0; t < 3; ++t)
        LVA_TRY(lva_reorder_tokens(stage + size_t(t) * tensor_in + p0 * plane_in,
                                   tile + size_t(t) * tensor_tile + p0 * plane_tile, hn, sh->T, sh->Hg, sh->Wg,
                                   sh->tile_t, sh->tile_h, sh->tile_w, n_pad, d, 2, 0, compute));
      const void* q = tile + p0 * plane_tile;
      const void* k = tile + tensor_tile + p0 * plane_tile;
      const void* v = tile + 2 * tensor_tile + p0 * plane_tile;
      // per-head masks: the group's rows of the CSR (row_ptr holds absolute offsets)
      const int32_t* rp = mask->mask_heads == 1 ? bufs->row_ptr : bufs->row_ptr + int64_t(h0) * nb;
      const int mh = mask->mask_heads == 1 ? 1 : hn;
      float* lse = bufs->lse_stage + p0 * n_pad;
      if (query_src == nullptr) {
        LVA_TRY(lva_block_sparse_attn_raster(q, k, v, o_st + p0 * plane_in, lse, 1, hn, n_pad, N, d, bs, rp,
                                             bufs->col_idx, bufs->col_len, mh, sh->scale, sh->T, sh->Hg, sh->Wg,
                                             sh->tile_t, sh->tile_h, sh->tile_w, compute));
      } else {
        // repetitive heads: anchors in tile order, broadcast, then the inverse reorder
        char* ot = static_cast<char*>(bufs->o_tile) + p0 * plane_tile;
        const int32_t* qs = src_heads == 1 ? query_src : query_src + int64_t(h0) * nb;
        const int sh_n = src_heads == 1 ? 1 : hn;
        LVA_TRY(lva_block_sparse_attn(q, k, v, ot, lse, 1, hn, n_pad, N, d, bs, rp, bufs->col_idx, bufs->col_len,
                                      mh, sh->scale, qs, sh_n, compute));
        LVA_TRY(lva_broadcast_blocks(ot, lse, 1, hn, n_pad, d, bs, qs, sh_n, compute));
        LVA_TRY(lva_reorder_tokens(ot, o_st + p0 * plane_in, hn, sh->T, sh->Hg, sh->Wg, sh->tile_t, sh->tile_h,
                                   sh->tile_w, n_pad, d, 2, 1, compute));
      }
    }
    LVA_TRY(cuda(cudaEventRecord(ev[groups + g], compute), "record"));
  }
  LVA_TRY(cuda(cudaEventRecord(staging_free, compute), "record"));

  // --- device to host, per group, as each group's compute completes
  char* o_h = static_cast<char*>(o_host);
  for (int g = 0; g < groups; ++g) {
    const int b = g / per_b, h0 = (g % per_b) * heads, h1 = h0 + heads < H ? h0 + heads : H;
    if (h0 >= H) continue;
    const size_t p0 = size_t(b) * H + h0, hn = size_t(h1 - h0);
    LVA_TRY(cuda(cudaStreamWaitEvent(d2h, ev[groups + g], 0), "wait compute"));
    LVA_TRY(cuda(cudaMemcpyAsync(o_h + p0 * plane_in, o_st + p0 * plane_in, hn * plane_in, cudaMemcpyDeviceToHost, d2h),
                 "copy out"));
    LVA_TRY(cuda(cudaMemcpyAsync(lse_host + p0 * n_pad, bufs->lse_stage + p0 * n_pad, hn * size_t(n_pad) * 4,
                                 cudaMemcpyDeviceToHost, d2h), "copy out"));
  }
  LVA_TRY(cuda(cudaEventRecord(out_free, d2h), "record"));
#undef LVA_TRY
  if (done != nullptr) *done = out_free;
  return set_error_message(LVA_OK, "");
}

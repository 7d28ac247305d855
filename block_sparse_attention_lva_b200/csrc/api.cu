// api.cu -- the C ABI declared in include/lva.h: argument checks, status codes, the
// per-thread error message, the per-device kernel error word, and dispatch to launchers.
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "kernels.h"
#include "lva.h"

namespace lva {
namespace {

thread_local char g_msg[256] = "";

lva_status fail(lva_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

lva_status ok() {
  g_msg[0] = '\0';
  return LVA_OK;
}

lva_status from_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(LVA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Kernel-side error word: [0] = status, [1] = detail, read and written as one 64-bit word.
// One copy per device (module global); its device address is looked up once per device (on
// every call past the cache).
__device__ __align__(8) int g_device_error[2];

// Where lva_device_error's exchange kernel leaves the word it took.
__device__ unsigned long long g_device_error_taken;

// Takes the error word and clears it in one atomic exchange, so a fault recorded by a
// kernel on another stream at the same moment is either taken now or left for the next
// read, never lost.
__global__ void take_error_kernel(unsigned long long* word) {
  g_device_error_taken = atomicExch(word, 0ull);
}

// lva_device_error calls are serialised: they share the taken-word slot of a device.
std::mutex g_take_mutex;

std::atomic<int*> g_err_ptr[kMaxCachedDevices] = {};

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

lva_status set_error_message(lva_status status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return status;
}

int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  const bool cacheable = dev >= 0 && dev < kMaxCachedDevices;
  if (cacheable) {
    int* cached = g_err_ptr[dev].load(std::memory_order_acquire);
    if (cached != nullptr) return cached;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  if (cacheable) g_err_ptr[dev].store(static_cast<int*>(p), std::memory_order_release);
  return static_cast<int*>(p);
}

}  // namespace lva

using namespace lva;

extern "C" {

const char* lva_status_string(lva_status s) {
  switch (s) {
    case LVA_OK: return "LVA_OK";
    case LVA_ERR_INVALID_ARG: return "LVA_ERR_INVALID_ARG";
    case LVA_ERR_UNSUPPORTED: return "LVA_ERR_UNSUPPORTED";
    case LVA_ERR_CAPACITY: return "LVA_ERR_CAPACITY";
    case LVA_ERR_CUDA: return "LVA_ERR_CUDA";
    case LVA_ERR_TIMEOUT: return "LVA_ERR_TIMEOUT";
  }
  return "LVA_ERR_UNKNOWN";
}

const char* lva_last_error_message(void) { return g_msg; }

int lva_version(void) { return LVA_VERSION; }

lva_status lva_reorder_tokens(const void* src, void* dst, int64_t planes, int T, int H, int W,
                              int tile_t, int tile_h, int tile_w, int64_t n_pad, int64_t row_elems,
                              int elem_bytes, int inverse, cudaStream_t stream) {
  if (planes < 0) return fail(LVA_ERR_INVALID_ARG, "reorder: planes < 0");
  if (T <= 0 || H <= 0 || W <= 0 || tile_t <= 0 || tile_h <= 0 || tile_w <= 0)
    return fail(LVA_ERR_INVALID_ARG, "reorder: grid and tile sizes must be positive");
  if (elem_bytes != 2 && elem_bytes != 4) return fail(LVA_ERR_INVALID_ARG, "reorder: elem_bytes must be 2 or 4");
  if (row_elems <= 0) return fail(LVA_ERR_INVALID_ARG, "reorder: row_elems must be positive");
  const int64_t n = int64_t(T) * H * W;
  if (n >= (int64_t(1) << 31)) return fail(LVA_ERR_UNSUPPORTED, "reorder: T*H*W must be < 2^31");
  if (n_pad < n || n_pad >= (int64_t(1) << 31)) return fail(LVA_ERR_INVALID_ARG, "reorder: need T*H*W <= n_pad < 2^31");
  const int64_t row_bytes = row_elems * elem_bytes;
  if (row_bytes > (int64_t(1) << 20)) return fail(LVA_ERR_UNSUPPORTED, "reorder: rows above 1 MiB");
  // One thread per (row, chunk); chunks are at least elem_bytes wide, and the launch's
  // blocks of 256 threads must fit gridDim.x.
  if ((n_pad * row_elems + 255) / 256 > int64_t(0x7fffffff))
    return fail(LVA_ERR_UNSUPPORTED, "reorder: n_pad * row_elems too large for one launch");
  if (planes == 0) return ok();
  if (src == nullptr || dst == nullptr) return fail(LVA_ERR_INVALID_ARG, "reorder: null pointer");
  if (!aligned(src, elem_bytes) || !aligned(dst, elem_bytes))
    return fail(LVA_ERR_INVALID_ARG, "reorder: pointers must be aligned to elem_bytes");
  ReorderArgs a{src, dst, planes, T, H, W, tile_t, tile_h, tile_w, n, n_pad, row_bytes, inverse != 0};
  return from_cuda(launch_reorder(a, stream), "reorder launch");
}

static lva_status check_mask_params(const lva_mask_params* p) {
  if (p == nullptr) return fail(LVA_ERR_INVALID_ARG, "mask: null params");
  if (p->block_size != 64 && p->block_size != 128) return fail(LVA_ERR_UNSUPPORTED, "mask: block_size must be 64 or 128");
  if (p->n_pad <= 0 || p->n_pad % p->block_size != 0) return fail(LVA_ERR_INVALID_ARG, "mask: n_pad must be a positive multiple of block_size");
  if (p->n_valid < 1 || p->n_valid > p->n_pad) return fail(LVA_ERR_INVALID_ARG, "mask: need 1 <= n_valid <= n_pad");
  if (p->mask_heads < 1) return fail(LVA_ERR_INVALID_ARG, "mask: mask_heads must be >= 1");
  const int64_t nb = p->n_pad / p->block_size;
  if (int64_t(p->mask_heads) * nb * nb >= (int64_t(1) << 31))
    return fail(LVA_ERR_UNSUPPORTED, "mask: mask_heads*nb*nb must be < 2^31");
  switch (p->kind) {
    case LVA_MASK_WINDOW_ANCHOR:
      if (p->window_unit_tokens < 1 || p->window_radius < 0 || p->num_anchors < 0 || p->step < 0)
        return fail(LVA_ERR_INVALID_ARG, "mask: window needs unit >= 1, radius >= 0, anchors >= 0, step >= 0");
      if (p->num_anchors > nb) return fail(LVA_ERR_INVALID_ARG, "mask: more anchors than blocks");
      if (p->mask_heads != 1) return fail(LVA_ERR_INVALID_ARG, "mask: parametric kinds build one mask head");
      break;
    case LVA_MASK_TWO_STAGE:
      if (p->group_blocks < 1) return fail(LVA_ERR_INVALID_ARG, "mask: group_blocks must be >= 1");
      if (p->mask_heads != 1) return fail(LVA_ERR_INVALID_ARG, "mask: parametric kinds build one mask head");
      break;
    case LVA_MASK_ALL:
      if (p->mask_heads != 1) return fail(LVA_ERR_INVALID_ARG, "mask: parametric kinds build one mask head");
      break;
    case LVA_MASK_LVSA_FRAMES: {
      if (p->window_unit_tokens < 1 || p->num_anchors < 0 || p->step < 0 || p->budget_frames < 1)
        return fail(LVA_ERR_INVALID_ARG, "mask: LVSA frames need unit >= 1, anchors >= 0, step >= 0, budget >= 1");
      const int64_t frames = (p->n_valid + p->window_unit_tokens - 1) / p->window_unit_tokens;
      if (p->num_anchors > frames) return fail(LVA_ERR_INVALID_ARG, "mask: more global frames than frames");
      if (p->mask_heads != 1) return fail(LVA_ERR_INVALID_ARG, "mask: parametric kinds build one mask head");
      break;
    }
    case LVA_MASK_STATIC:
      break;
    default:
      return fail(LVA_ERR_INVALID_ARG, "mask: unknown kind %d", p->kind);
  }
  return ok();
}

int64_t lva_block_mask_max_nnz(const lva_mask_params* p) {
  if (check_mask_params(p) != LVA_OK) return 0;
  const int64_t nb = p->n_pad / p->block_size;
  return int64_t(p->mask_heads) * nb * nb;
}

// Checks shared by both mask-build calls; fills the launcher arguments.
static lva_status mask_args(const lva_mask_params* p, const uint8_t* dense_mask, int32_t* row_ptr,
                            int32_t* col_idx, int64_t col_capacity, int32_t* nnz_out, MaskArgs* a) {
  lva_status s = check_mask_params(p);
  if (s != LVA_OK) return s;
  if (row_ptr == nullptr || col_idx == nullptr || nnz_out == nullptr)
    return fail(LVA_ERR_INVALID_ARG, "mask: null output pointer");
  if (!aligned(row_ptr, 4) || !aligned(col_idx, 4) || !aligned(nnz_out, 4))
    return fail(LVA_ERR_INVALID_ARG, "mask: outputs must be 4-byte aligned");
  if (p->kind == LVA_MASK_STATIC && dense_mask == nullptr)
    return fail(LVA_ERR_INVALID_ARG, "mask: STATIC needs dense_mask");
  const int64_t need = lva_block_mask_max_nnz(p);
  if (col_capacity < need)
    return fail(LVA_ERR_CAPACITY, "mask: col_capacity %lld < %lld", (long long)col_capacity, (long long)need);
  a->kind = p->kind;
  a->mask_heads = p->mask_heads;
  a->block_size = p->block_size;
  a->n_pad = p->n_pad;
  a->n_valid = p->n_valid;
  a->unit_tokens = p->window_unit_tokens;
  a->radius = p->window_radius;
  a->num_anchors = p->num_anchors;
  a->step = p->step;
  a->group_blocks = p->group_blocks;
  a->budget_frames = p->budget_frames;
  a->dense = dense_mask;
  a->row_ptr = row_ptr;
  a->col_idx = col_idx;
  a->nnz_out = nnz_out;
  return LVA_OK;
}

lva_status lva_build_block_mask(const lva_mask_params* p, const uint8_t* dense_mask, int32_t* row_ptr,
                                int32_t* col_idx, int64_t col_capacity, int32_t* nnz_out,
                                cudaStream_t stream) {
  MaskArgs a;
  const lva_status s = mask_args(p, dense_mask, row_ptr, col_idx, col_capacity, nnz_out, &a);
  if (s != LVA_OK) return s;
  return from_cuda(launch_build_mask(a, stream), "mask launch");
}

int64_t lva_block_mask_workspace_bytes(const lva_mask_params* p) {
  if (check_mask_params(p) != LVA_OK) return -1;
  const int64_t nb = p->n_pad / p->block_size;
  return mask_workspace_bytes(p->kind, int64_t(p->mask_heads) * nb, nb);
}

lva_status lva_build_block_mask_ws(const lva_mask_params* p, const uint8_t* dense_mask, int32_t* row_ptr,
                                   int32_t* col_idx, int64_t col_capacity, int32_t* nnz_out, void* workspace,
                                   int64_t workspace_bytes, cudaStream_t stream) {
  MaskArgs a;
  const lva_status s = mask_args(p, dense_mask, row_ptr, col_idx, col_capacity, nnz_out, &a);
  if (s != LVA_OK) return s;
  const int64_t need = lva_block_mask_workspace_bytes(p);
  if (need == 0) return from_cuda(launch_build_mask(a, stream), "mask launch");
  if (workspace == nullptr) return fail(LVA_ERR_INVALID_ARG, "mask: null workspace");
  if (!aligned(workspace, 16)) return fail(LVA_ERR_INVALID_ARG, "mask: workspace must be 16-byte aligned");
  if (workspace_bytes < need)
    return fail(LVA_ERR_CAPACITY, "mask: workspace_bytes %lld < %lld", (long long)workspace_bytes, (long long)need);
  return from_cuda(launch_build_mask_packed(a, workspace, stream), "mask launch");
}

lva_status lva_build_block_mask_noalloc(const lva_mask_params* p, const uint8_t* dense_mask, int32_t* row_ptr,
                                        int32_t* col_idx, int64_t col_capacity, int32_t* nnz_out,
                                        cudaStream_t stream) {
  MaskArgs a;
  const lva_status s = mask_args(p, dense_mask, row_ptr, col_idx, col_capacity, nnz_out, &a);
  if (s != LVA_OK) return s;
  const int64_t need = lva_block_mask_workspace_bytes(p);
  if (need > mask_noalloc_scratch_bytes())
    return fail(LVA_ERR_CAPACITY,
                "mask_noalloc: these parameters need %lld bytes of scratch; the library holds %lld "
                "(use lva_build_block_mask_ws with a workspace, or lva_build_block_mask)",
                (long long)need, (long long)mask_noalloc_scratch_bytes());
  return from_cuda(launch_build_mask_noalloc(a, stream), "mask_noalloc launch");
}

static lva_status attn_common(const char* fn, const void* q, const void* k, const void* v, void* o,
                              float* lse, int B, int H, int64_t n_pad, int64_t n_valid, int d,
                              int block_size, const int32_t* row_ptr, const int32_t* col_idx,
                              int64_t col_len, int mask_heads, float scale, const int32_t* query_src,
                              int src_heads, void* o_raster, int T, int Hg, int Wg, int tile_t,
                              int tile_h, int tile_w, int gather_windows, int gather_window,
                              cudaStream_t stream, int lse_only = 0) {
  if (B < 0 || H < 1) return fail(LVA_ERR_INVALID_ARG, "%s: need B >= 0 and H >= 1", fn);
  if (d != 64 && d != 128) return fail(LVA_ERR_UNSUPPORTED, "%s: head dim must be 64 or 128", fn);
  if (block_size != 64 && block_size != 128) return fail(LVA_ERR_UNSUPPORTED, "%s: block_size must be 64 or 128", fn);
  if (n_pad <= 0 || n_pad % block_size != 0) return fail(LVA_ERR_INVALID_ARG, "%s: n_pad must be a positive multiple of block_size", fn);
  if (n_valid < 0 || n_valid > n_pad) return fail(LVA_ERR_INVALID_ARG, "%s: need 0 <= n_valid <= n_pad", fn);
  if (mask_heads != 1 && mask_heads != H) return fail(LVA_ERR_INVALID_ARG, "%s: mask_heads must be 1 or H", fn);
  if (int64_t(B) * H * n_pad >= (int64_t(1) << 31)) return fail(LVA_ERR_UNSUPPORTED, "%s: B*H*n_pad must be < 2^31", fn);
  if (!(scale == scale)) return fail(LVA_ERR_INVALID_ARG, "%s: scale is NaN", fn);
  if (col_len < 0) return fail(LVA_ERR_INVALID_ARG, "%s: col_len < 0", fn);
  if (query_src != nullptr && src_heads != 1 && src_heads != H)
    return fail(LVA_ERR_INVALID_ARG, "%s: src_heads must be 1 or H", fn);
  if (query_src != nullptr && !aligned(query_src, 4))
    return fail(LVA_ERR_INVALID_ARG, "%s: query_src must be 4-byte aligned", fn);
  if (o_raster != nullptr) {
    if (T < 1 || Hg < 1 || Wg < 1 || tile_t < 1 || tile_h < 1 || tile_w < 1)
      return fail(LVA_ERR_INVALID_ARG, "%s: grid and tile extents must be >= 1", fn);
    if (int64_t(T) * Hg * Wg != n_valid)
      return fail(LVA_ERR_INVALID_ARG, "%s: T*H*W must equal n_valid", fn);
  }
  if (B == 0) return ok();
  if (!q || !k || (!lse_only && (!v || !(o || o_raster))) || !lse || !row_ptr || (!col_idx && col_len > 0))
    return fail(LVA_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!aligned(q, 16) || !aligned(k, 16) || (v && !aligned(v, 16)) || (o && !aligned(o, 16)) ||
      (o_raster && !aligned(o_raster, 16)))
    return fail(LVA_ERR_INVALID_ARG, "%s: q, k, v, o must be 16-byte aligned", fn);
  if (!aligned(lse, 4) || !aligned(row_ptr, 4) || !aligned(col_idx, 4))
    return fail(LVA_ERR_INVALID_ARG, "%s: lse, row_ptr, col_idx must be 4-byte aligned", fn);
  int* err = device_error_word();
  if (err == nullptr) return fail(LVA_ERR_CUDA, "%s: cannot locate the device error word", fn);
  AttnArgs a{q, k, v, o, lse, B, H, n_pad, n_valid, d, block_size, row_ptr,
             col_idx, col_len, mask_heads, scale, query_src, src_heads, err,
             o_raster, T, Hg, Wg, tile_t, tile_h, tile_w, gather_windows, gather_window, lse_only};
  const char* why = "launch";
  cudaError_t e = launch_attn(a, stream, &why);
  if (e != cudaSuccess) return fail(LVA_ERR_CUDA, "%s: %s: %s", fn, why, cudaGetErrorString(e));
  return ok();
}

lva_status lva_block_sparse_attn(const void* q, const void* k, const void* v, void* o, float* lse,
                                 int B, int H, int64_t n_pad, int64_t n_valid, int d, int block_size,
                                 const int32_t* row_ptr, const int32_t* col_idx, int64_t col_len,
                                 int mask_heads, float scale, const int32_t* query_src, int src_heads,
                                 cudaStream_t stream) {
  if (o == nullptr && B > 0) return fail(LVA_ERR_INVALID_ARG, "attn: null pointer");
  return attn_common("attn", q, k, v, o, lse, B, H, n_pad, n_valid, d, block_size, row_ptr, col_idx,
                     col_len, mask_heads, scale, query_src, src_heads, nullptr, 0, 0, 0, 0, 0, 0, 0, 0,
                     stream);
}

lva_status lva_block_sparse_lse(const void* q, const void* k, float* lse, int B, int H, int64_t n_pad,
                                int64_t n_valid, int d, int block_size, const int32_t* row_ptr,
                                const int32_t* col_idx, int64_t col_len, int mask_heads, float scale,
                                cudaStream_t stream) {
  return attn_common("lse", q, k, nullptr, nullptr, lse, B, H, n_pad, n_valid, d, block_size, row_ptr,
                     col_idx, col_len, mask_heads, scale, nullptr, 1, nullptr, 0, 0, 0, 0, 0, 0, 0, 0,
                     stream, 1);
}

lva_status lva_block_sparse_attn_raster(const void* q, const void* k, const void* v, void* o_raster,
                                        float* lse, int B, int H, int64_t n_pad, int64_t n_valid,
                                        int d, int block_size, const int32_t* row_ptr,
                                        const int32_t* col_idx, int64_t col_len, int mask_heads,
                                        float scale, int T, int Hg, int Wg, int tile_t, int tile_h,
                                        int tile_w, cudaStream_t stream) {
  if (o_raster == nullptr && B > 0) return fail(LVA_ERR_INVALID_ARG, "attn_raster: null pointer");
  return attn_common("attn_raster", q, k, v, nullptr, lse, B, H, n_pad, n_valid, d, block_size,
                     row_ptr, col_idx, col_len, mask_heads, scale, nullptr, 1, o_raster, T, Hg, Wg,
                     tile_t, tile_h, tile_w, 0, 0, stream);
}

lva_status lva_window_transposed_attn(const void* q, const void* k, const void* v, void* o, float* lse,
                                      int B, int H, int64_t n, int d, int window, int block_size,
                                      const int32_t* row_ptr, const int32_t* col_idx, int64_t col_len,
                                      int mask_heads, float scale, cudaStream_t stream) {
  if (window < 1 || n <= 0 || n % window != 0)
    return fail(LVA_ERR_INVALID_ARG, "window_attn: n must be a positive multiple of window");
  const int64_t m = n / window;
  if (block_size != 64 && block_size != 128)
    return fail(LVA_ERR_UNSUPPORTED, "window_attn: block_size must be 64 or 128");
  if (m % block_size != 0)
    return fail(LVA_ERR_INVALID_ARG, "window_attn: the window count n / window must be a multiple of block_size");
  if (int64_t(B) * H * m >= (int64_t(1) << 31))
    return fail(LVA_ERR_UNSUPPORTED, "window_attn: B*H*(n/window) must be < 2^31");
  if (o == nullptr && B > 0) return fail(LVA_ERR_INVALID_ARG, "window_attn: null pointer");
  // O goes to the original order through the raster epilogue: the window transpose is the
  // tile order of the grid (1, m, window) with tiles (1, m, 1).
  return attn_common("window_attn", q, k, v, nullptr, lse, B, H, n, n, d, block_size, row_ptr, col_idx,
                     col_len, mask_heads, scale, nullptr, 1, o, 1, int(m), window, 1, int(m), 1, int(m),
                     window, stream);
}

lva_status lva_broadcast_blocks(void* o, float* lse, int B, int H, int64_t n_pad, int d, int block_size,
                                const int32_t* query_src, int src_heads, cudaStream_t stream) {
  if (B < 0 || H < 1) return fail(LVA_ERR_INVALID_ARG, "broadcast: need B >= 0 and H >= 1");
  if (d != 64 && d != 128) return fail(LVA_ERR_UNSUPPORTED, "broadcast: head dim must be 64 or 128");
  if (block_size != 64 && block_size != 128) return fail(LVA_ERR_UNSUPPORTED, "broadcast: block_size must be 64 or 128");
  if (n_pad <= 0 || n_pad % block_size != 0) return fail(LVA_ERR_INVALID_ARG, "broadcast: n_pad must be a positive multiple of block_size");
  if (src_heads != 1 && src_heads != H) return fail(LVA_ERR_INVALID_ARG, "broadcast: src_heads must be 1 or H");
  if (int64_t(B) * H * n_pad >= (int64_t(1) << 31)) return fail(LVA_ERR_UNSUPPORTED, "broadcast: B*H*n_pad must be < 2^31");
  if (B == 0) return ok();
  if (!o || !lse || !query_src) return fail(LVA_ERR_INVALID_ARG, "broadcast: null pointer");
  if (!aligned(o, 16) || !aligned(lse, 4) || !aligned(query_src, 4))
    return fail(LVA_ERR_INVALID_ARG, "broadcast: o must be 16-byte, lse and query_src 4-byte aligned");
  int* err = device_error_word();
  if (err == nullptr) return fail(LVA_ERR_CUDA, "broadcast: cannot locate the device error word");
  BroadcastArgs a{o, lse, B, H, n_pad, d, block_size, query_src, src_heads, err};
  return from_cuda(launch_broadcast(a, stream), "broadcast launch");
}

lva_status lva_block_energy(const void* q, const void* k, const float* lse, float* energy, int B,
                            int H, int64_t n_pad, int64_t n_valid, int d, int block_size,
                            const int32_t* row_ptr, const int32_t* col_idx, int64_t col_len,
                            int mask_heads, float scale, cudaStream_t stream) {
  if (B < 0 || H < 1) return fail(LVA_ERR_INVALID_ARG, "energy: need B >= 0 and H >= 1");
  if (d != 64 && d != 128) return fail(LVA_ERR_UNSUPPORTED, "energy: head dim must be 64 or 128");
  if (block_size != 64 && block_size != 128) return fail(LVA_ERR_UNSUPPORTED, "energy: block_size must be 64 or 128");
  if (n_pad <= 0 || n_pad % block_size != 0) return fail(LVA_ERR_INVALID_ARG, "energy: n_pad must be a positive multiple of block_size");
  if (n_valid < 0 || n_valid > n_pad) return fail(LVA_ERR_INVALID_ARG, "energy: need 0 <= n_valid <= n_pad");
  if (mask_heads != 1 && mask_heads != H) return fail(LVA_ERR_INVALID_ARG, "energy: mask_heads must be 1 or H");
  if (int64_t(B) * H * n_pad >= (int64_t(1) << 31)) return fail(LVA_ERR_UNSUPPORTED, "energy: B*H*n_pad must be < 2^31");
  if (!(scale == scale)) return fail(LVA_ERR_INVALID_ARG, "energy: scale is NaN");
  if (col_len < 0) return fail(LVA_ERR_INVALID_ARG, "energy: col_len < 0");
  if (B == 0) return ok();
  if (!q || !k || !lse || !energy || !row_ptr || (!col_idx && col_len > 0))
    return fail(LVA_ERR_INVALID_ARG, "energy: null pointer");
  if (!aligned(q, 16) || !aligned(k, 16))
    return fail(LVA_ERR_INVALID_ARG, "energy: q, k must be 16-byte aligned");
  if (!aligned(lse, 4) || !aligned(energy, 4) || !aligned(row_ptr, 4) || !aligned(col_idx, 4))
    return fail(LVA_ERR_INVALID_ARG, "energy: lse, energy, row_ptr, col_idx must be 4-byte aligned");
  int* err = device_error_word();
  if (err == nullptr) return fail(LVA_ERR_CUDA, "energy: cannot locate the device error word");
  EnergyArgs a{q, k, lse, energy, B, H, n_pad, n_valid, d, block_size, row_ptr, col_idx, col_len,
               mask_heads, scale, err};
  const char* why = "launch";
  cudaError_t e = launch_energy(a, stream, &why);
  if (e != cudaSuccess) return fail(LVA_ERR_CUDA, "energy: %s: %s", why, cudaGetErrorString(e));
  return ok();
}

lva_status lva_select_blocks(const float* energy, uint8_t* mask, int64_t rows, int nb, double eps,
                             cudaStream_t stream) {
  if (rows < 0) return fail(LVA_ERR_INVALID_ARG, "select: rows < 0");
  if (nb < 1) return fail(LVA_ERR_INVALID_ARG, "select: nb must be >= 1");
  if (nb > kSelectMaxBlocks) return fail(LVA_ERR_UNSUPPORTED, "select: nb must be <= %d", kSelectMaxBlocks);
  if (!(eps >= 0.0 && eps <= 1.0)) return fail(LVA_ERR_INVALID_ARG, "select: eps must be in [0, 1]");
  if (rows > (int64_t(1) << 40) / nb) return fail(LVA_ERR_UNSUPPORTED, "select: rows * nb too large");
  if (rows == 0) return ok();
  if (!energy || !mask) return fail(LVA_ERR_INVALID_ARG, "select: null pointer");
  if (!aligned(energy, 4)) return fail(LVA_ERR_INVALID_ARG, "select: energy must be 4-byte aligned");
  int* err = device_error_word();
  if (err == nullptr) return fail(LVA_ERR_CUDA, "select: cannot locate the device error word");
  SelectArgs a{energy, mask, rows, nb, eps, err};
  return from_cuda(launch_select(a, stream), "select launch");
}

lva_status lva_aggregate_masks(const uint8_t* masks, uint8_t* out, int prompts, int64_t count,
                               double rho, cudaStream_t stream) {
  if (prompts < 1) return fail(LVA_ERR_INVALID_ARG, "aggregate: prompts must be >= 1");
  if (count < 0) return fail(LVA_ERR_INVALID_ARG, "aggregate: count < 0");
  if (!(rho >= 0.0 && rho <= 1.0)) return fail(LVA_ERR_INVALID_ARG, "aggregate: rho must be in [0, 1]");
  if (count == 0) return ok();
  if (!masks || !out) return fail(LVA_ERR_INVALID_ARG, "aggregate: null pointer");
  AggregateArgs a{masks, out, prompts, count, rho * double(prompts)};
  return from_cuda(launch_aggregate(a, stream), "aggregate launch");
}

lva_status lva_selftest_wait(int mode, cudaStream_t stream) {
  if (mode < 0 || mode > 2) return fail(LVA_ERR_INVALID_ARG, "selftest_wait: mode must be 0, 1 or 2");
  int* err = device_error_word();
  if (err == nullptr) return fail(LVA_ERR_CUDA, "selftest_wait: cannot locate the device error word");
  return from_cuda(launch_wait_selftest(mode, err, stream), "selftest_wait launch");
}

lva_status lva_device_error(cudaStream_t stream, lva_status* status, int* detail) {
  if (status == nullptr) return fail(LVA_ERR_INVALID_ARG, "device_error: null status");
  int* err = device_error_word();
  if (err == nullptr) return fail(LVA_ERR_CUDA, "device_error: cannot locate the device error word");
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return from_cuda(e, "device_error: stream sync");
  unsigned long long word = 0;
  {
    std::lock_guard<std::mutex> lock(g_take_mutex);
    take_error_kernel<<<1, 1, 0, stream>>>(reinterpret_cast<unsigned long long*>(err));
    e = cudaGetLastError();
    if (e != cudaSuccess) return from_cuda(e, "device_error: exchange launch");
    e = cudaMemcpyFromSymbolAsync(&word, g_device_error_taken, sizeof(word), 0, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return from_cuda(e, "device_error: read");
  }
  *status = static_cast<lva_status>(static_cast<int>(word & 0xffffffffull));
  if (detail) *detail = static_cast<int>(word >> 32);
  return ok();
}

}  // extern "C"

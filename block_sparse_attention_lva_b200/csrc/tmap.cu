// tmap.cu -- TMA tensor maps for the kernels that stream bf16 [rows, d] tiles.
//
// cuTensorMapEncodeTiled is a driver API function; it is fetched through the runtime's
// driver entry point query, so the library links only the static CUDA runtime.
#include <cuda.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace lva {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lookup_encode_tiled() {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<EncodeTiledFn>(ptr);
  return nullptr;
}

// Looked up once; the initialisation of a function-local static is thread-safe, so
// concurrent first calls from several host threads do not race.
EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = lookup_encode_tiled();
  return fn;
}

}  // namespace

bool make_rows_map(CUtensorMap* m, const void* base, int64_t rows, int d, int box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(d) * 2};
  const cuuint32_t box[2] = {64u, cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_window_gather_map(CUtensorMap* m, const void* base, int64_t planes, int windows, int window,
                            int d, int box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  // [planes * windows, window, d] viewed innermost-first: element x of position p of window
  // a' = plane * windows + a sits at ((a' * window) + p) * d + x.
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(window), cuuint64_t(planes * windows)};
  const cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(window) * cuuint64_t(d) * 2};
  const cuuint32_t box[3] = {64u, 1u, cuuint32_t(box_rows)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace lva

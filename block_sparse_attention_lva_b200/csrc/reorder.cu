// reorder.cu -- spatiotemporal-tile token permutation (gather) and its inverse (scatter).
//
// Token order: tiles of tt x th x tw latent tokens in raster order of tile coordinates,
// tokens in raster order inside a tile, edge tiles partial.  The tile-order position k is
// turned into its raster index in closed form (no table), then whole rows are copied with
// 16-byte (or narrower) vector accesses.  The permutation does not depend on the plane
// (batch x head), so each thread computes it once and copies that row for every plane.
//
// HBM-bound: a forward pass reads N rows and writes n_pad rows per plane.
#include <cstdint>

#include "kernels.h"
#include "tile_order.cuh"

namespace lva {
namespace {

template <int CHUNK>
struct Vec;
template <> struct Vec<16> { using T = int4; };
template <> struct Vec<8> { using T = int2; };
template <> struct Vec<4> { using T = int; };
template <> struct Vec<2> { using T = short; };

constexpr int kThreads = 256;
constexpr int kPlaneUnroll = 4;

// One thread per (row k, chunk c); loops over planes.  Forward: k in [0, n_pad),
// reads src row perm[k] (raster) and writes dst row k (tile order); rows >= N are zeroed.
// Inverse: k in [0, N), reads src row k (tile order), writes dst row perm[k] (raster).
template <int CHUNK>
__global__ void __launch_bounds__(kThreads) reorder_kernel(
    const char* __restrict__ src, char* __restrict__ dst, int64_t planes, Grid3 g,
    uint32_t n_valid, uint32_t rows, uint32_t chunks_per_row, int64_t src_plane_bytes,
    int64_t dst_plane_bytes, int inverse) {
  using V = typename Vec<CHUNK>::T;
  const uint64_t idx = static_cast<uint64_t>(blockIdx.x) * kThreads + threadIdx.x;
  if (idx >= static_cast<uint64_t>(rows) * chunks_per_row) return;
  const uint32_t k = static_cast<uint32_t>(idx / chunks_per_row);
  const uint32_t c = static_cast<uint32_t>(idx - static_cast<uint64_t>(k) * chunks_per_row);
  const int64_t row_bytes = static_cast<int64_t>(chunks_per_row) * CHUNK;

  if (!inverse && k >= n_valid) {  // padding rows of the tile-order output
    const V zero{};
    for (int64_t p = 0; p < planes; ++p)
      __stcs(reinterpret_cast<V*>(dst + p * dst_plane_bytes + k * row_bytes) + c, zero);
    return;
  }
  const uint32_t raster = tile_order_to_raster(k, g);
  const int64_t src_off = (inverse ? int64_t(k) : int64_t(raster)) * row_bytes + int64_t(c) * CHUNK;
  const int64_t dst_off = (inverse ? int64_t(raster) : int64_t(k)) * row_bytes + int64_t(c) * CHUNK;

  int64_t p = 0;
  for (; p + kPlaneUnroll <= planes; p += kPlaneUnroll) {
    V v[kPlaneUnroll];
#pragma unroll
    for (int u = 0; u < kPlaneUnroll; ++u)
      v[u] = __ldcs(reinterpret_cast<const V*>(src + (p + u) * src_plane_bytes + src_off));
#pragma unroll
    for (int u = 0; u < kPlaneUnroll; ++u)
      __stcs(reinterpret_cast<V*>(dst + (p + u) * dst_plane_bytes + dst_off), v[u]);
  }
  for (; p < planes; ++p) {
    V v = __ldcs(reinterpret_cast<const V*>(src + p * src_plane_bytes + src_off));
    __stcs(reinterpret_cast<V*>(dst + p * dst_plane_bytes + dst_off), v);
  }
}

template <int CHUNK>
cudaError_t launch_chunk(const ReorderArgs& a, cudaStream_t stream) {
  Grid3 g{uint32_t(a.T), uint32_t(a.H), uint32_t(a.W), uint32_t(a.tt), uint32_t(a.th),
          uint32_t(a.tw)};
  const uint32_t rows = uint32_t(a.inverse ? a.n_valid : a.n_pad);
  const uint32_t cpr = uint32_t(a.row_bytes / CHUNK);
  const uint64_t threads = uint64_t(rows) * cpr;
  const uint64_t blocks = (threads + kThreads - 1) / kThreads;
  if (blocks == 0 || a.planes == 0) return cudaSuccess;
  const int64_t src_plane = (a.inverse ? a.n_pad : a.n_valid) * a.row_bytes;
  const int64_t dst_plane = (a.inverse ? a.n_valid : a.n_pad) * a.row_bytes;
  reorder_kernel<CHUNK><<<dim3(uint32_t(blocks)), kThreads, 0, stream>>>(
      static_cast<const char*>(a.src), static_cast<char*>(a.dst), a.planes, g,
      uint32_t(a.n_valid), rows, cpr, src_plane, dst_plane, a.inverse);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_reorder(const ReorderArgs& a, cudaStream_t stream) {
  const uintptr_t align = reinterpret_cast<uintptr_t>(a.src) | reinterpret_cast<uintptr_t>(a.dst);
  if (a.row_bytes % 16 == 0 && align % 16 == 0) return launch_chunk<16>(a, stream);
  if (a.row_bytes % 8 == 0 && align % 8 == 0) return launch_chunk<8>(a, stream);
  if (a.row_bytes % 4 == 0 && align % 4 == 0) return launch_chunk<4>(a, stream);
  return launch_chunk<2>(a, stream);
}

}  // namespace lva

// tile_order.cuh -- the spatiotemporal tile order of latent video tokens, in closed form.
//
// Tokens of a T x H x W latent grid are ordered by tiles of tt x th x tw tokens: tiles in
// raster order of their coordinates, tokens in raster order inside a tile, edge tiles
// partial (not padded), so that a run of Bs consecutive tokens is a spatiotemporal
// neighbourhood (the 3D blocks over which the LVSA and CalibAtt pages' block masks act).
// Used by the reorder kernels and by the attention epilogue that writes O in raster order.
#pragma once

#include <cstdint>

namespace lva {

__host__ __device__ __forceinline__ uint32_t umin_(uint32_t a, uint32_t b) { return a < b ? a : b; }

struct Grid3 {
  uint32_t T, H, W, tt, th, tw;
};

// Raster index of the k-th token in tile order (k < T*H*W).
__host__ __device__ __forceinline__ uint32_t tile_order_to_raster(uint32_t k, const Grid3& g) {
  const uint32_t hw = g.H * g.W;
  const uint32_t slab = g.tt * hw;                 // tokens in a full depth-tt slab
  const uint32_t it = k / slab;
  uint32_t r = k - it * slab;
  const uint32_t dt = umin_(g.tt, g.T - it * g.tt);  // depth of this slab (last may be short)
  const uint32_t row_tokens = dt * g.th * g.W;     // tokens in a full-height tile row
  const uint32_t ih = r / row_tokens;
  r -= ih * row_tokens;
  const uint32_t dh = umin_(g.th, g.H - ih * g.th);
  const uint32_t tile_tokens = dt * dh * g.tw;     // tokens in a full-width tile of this row
  const uint32_t iw = r / tile_tokens;
  r -= iw * tile_tokens;
  const uint32_t dw = umin_(g.tw, g.W - iw * g.tw);
  const uint32_t plane = dh * dw;
  const uint32_t t1 = r / plane;
  r -= t1 * plane;
  const uint32_t h1 = r / dw;
  const uint32_t w1 = r - h1 * dw;
  return (it * g.tt + t1) * hw + (ih * g.th + h1) * g.W + (iw * g.tw + w1);
}

}  // namespace lva

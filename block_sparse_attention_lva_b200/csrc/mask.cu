// mask.cu -- block mask -> per-query-block CSR, built on the GPU in three launches:
//   1. count: one warp per CSR row evaluates the mask predicate for 32 key blocks at a time
//      (or 512 bytes of a dense static mask) and reduces with ballot/popc; the count goes
//      to row_ptr[row + 1];
//   2. scan:  one CTA turns the counts into row offsets in place (inclusive scan of
//      row_ptr[1..R]) and writes nnz;
//   3. fill:  the count warp's pass again, writing each set column at its ballot rank.
// Rows come out in (mask head, query block) order with ascending, unique columns, which is
// a pure function of the parameters: the same CSR on every run.
#include <cstdint>

#include "kernels.h"

namespace lva {
namespace {

enum Kind { kWindowAnchor = 0, kStatic = 1, kAll = 2, kTwoStage = 3, kLvsaFrames = 4 };

struct MaskDev {
  int kind;
  int64_t nb;          // blocks per side
  int64_t rows;        // mask_heads * nb
  int64_t bs, n_valid, unit;
  int64_t radius;
  int64_t anchors, step;
  int64_t group;
  int64_t frames, budget;   // LVSA frames: T and C
  const uint8_t* dense;
};

// Window units spanned by the real tokens of block i (a padding-only block takes the unit
// of the last real token).
__device__ __forceinline__ void block_units(const MaskDev& m, int64_t i, int64_t& lo, int64_t& hi) {
  const int64_t first = i * m.bs;
  if (first >= m.n_valid) {
    lo = hi = (m.n_valid - 1) / m.unit;
  } else {
    lo = first / m.unit;
    hi = (min(first + m.bs, m.n_valid) - 1) / m.unit;
  }
}

// Is x one of the anchors {(floor(a*n/G) + s) mod n : a < G}?  (n = blocks or frames)
__device__ __forceinline__ bool is_anchor_of(int64_t x, int64_t n, int64_t G, int64_t s) {
  if (G <= 0) return false;
  const int64_t xx = ((x - s) % n + n) % n;
  // smallest a with floor(a*n/G) >= xx is ceil(xx*G/n)
  const int64_t a = (xx * G + n - 1) / n;
  return a < G && (a * n) / G == xx;
}

__device__ __forceinline__ bool is_anchor(const MaskDev& m, int64_t j) {
  return is_anchor_of(j, m.nb, m.anchors, m.step);
}

// LVSA expanded window of frame t: W grows from {t}, right then left alternately (the other
// side at a sequence end), until |G_s union W| = min(C, T).
__device__ __forceinline__ void lvsa_window(const MaskDev& m, int64_t t, int64_t& lo, int64_t& hi) {
  const int64_t T = m.frames;
  const int64_t target = min(m.budget, T);
  int64_t count = min(m.anchors, T) + (is_anchor_of(t, T, m.anchors, m.step) ? 0 : 1);
  lo = hi = t;
  bool right = true;
  while (count < target) {
    const bool can_r = hi + 1 < T, can_l = lo > 0;
    if (!can_r && !can_l) break;
    int64_t f;
    if ((right && can_r) || !can_l) f = ++hi; else f = --lo;
    if (!is_anchor_of(f, T, m.anchors, m.step)) ++count;
    right = !right;
  }
}

// Parametric predicate for rows of the non-static kinds.
__device__ __forceinline__ bool predicate(const MaskDev& m, int64_t i, int64_t j, int64_t lo_i,
                                          int64_t hi_i) {
  if (j >= m.nb) return false;
  switch (m.kind) {
    case kAll:
      return true;
    case kTwoStage:
      return (j / m.group == i / m.group) || (j == (i + m.group) % m.nb);
    case kLvsaFrames: {
      // lo_i / hi_i hold the union of the windows of i's frames
      int64_t lo_j, hi_j;
      block_units(m, j, lo_j, hi_j);
      if (lo_j <= hi_i && hi_j >= lo_i) return true;
      for (int64_t f = lo_j; f <= hi_j; ++f)
        if (is_anchor_of(f, m.frames, m.anchors, m.step)) return true;
      return false;
    }
    default: {
      int64_t lo_j, hi_j;
      block_units(m, j, lo_j, hi_j);
      const bool win = lo_j <= hi_i + m.radius && hi_j >= lo_i - m.radius;
      return win || is_anchor(m, j);
    }
  }
}

// Number of non-zero bytes in a 32-bit word.
__device__ __forceinline__ int nonzero_bytes(uint32_t w) {
  const uint32_t t = (((w & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w) & 0x80808080u;
  return __popc(t);
}

constexpr int kWarpsPerBlock = 8;

// Counts (FILL = false) or writes (FILL = true) the set columns of each row.
template <bool FILL>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) mask_rows_kernel(MaskDev m, int32_t* row_ptr,
                                                                     int32_t* col_idx) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  if (row >= m.rows) return;
  if (!FILL && row == 0 && lane == 0) row_ptr[0] = 0;
  const int64_t i = row % m.nb;
  int32_t base = FILL ? row_ptr[row] : 0;
  int32_t count = 0;

  if (m.kind == kStatic) {
    const uint8_t* src = m.dense + row * m.nb;
    const bool vec = (m.nb % 16 == 0) && ((reinterpret_cast<uintptr_t>(m.dense) & 15) == 0);
    if (vec) {
      // 16 bytes per lane, 512 key blocks per warp step.
      for (int64_t j0 = 0; j0 < m.nb; j0 += 512) {
        const int64_t j = j0 + lane * 16;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (j < m.nb) v = __ldcs(reinterpret_cast<const uint4*>(src + j));
        const int c = nonzero_bytes(v.x) + nonzero_bytes(v.y) + nonzero_bytes(v.z) + nonzero_bytes(v.w);
        if (FILL) {
          int incl = c;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
          }
          int pos = base + incl - c;
          const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int wv = 0; wv < 4; ++wv)
#pragma unroll
            for (int b = 0; b < 4; ++b)
              if ((words[wv] >> (8 * b)) & 0xFFu) col_idx[pos++] = static_cast<int32_t>(j + wv * 4 + b);
          base += __shfl_sync(0xffffffffu, incl, 31);
        } else {
          count += __reduce_add_sync(0xffffffffu, c);
        }
      }
    } else {
      for (int64_t j0 = 0; j0 < m.nb; j0 += 32) {
        const int64_t j = j0 + lane;
        const bool set = j < m.nb && src[j] != 0;
        const uint32_t ballot = __ballot_sync(0xffffffffu, set);
        if (FILL && set) col_idx[base + __popc(ballot & ((1u << lane) - 1u))] = static_cast<int32_t>(j);
        if (FILL) base += __popc(ballot); else count += __popc(ballot);
      }
    }
  } else {
    int64_t lo_i = 0, hi_i = 0;
    if (m.kind == kWindowAnchor) block_units(m, i, lo_i, hi_i);
    if (m.kind == kLvsaFrames) {
      // union of the (contiguous, overlapping) windows of the frames block i touches
      int64_t f0, f1;
      block_units(m, i, f0, f1);
      lo_i = m.frames;
      hi_i = -1;
      for (int64_t t = f0; t <= f1; ++t) {
        int64_t wl, wh;
        lvsa_window(m, t, wl, wh);
        lo_i = min(lo_i, wl);
        hi_i = max(hi_i, wh);
      }
    }
    for (int64_t j0 = 0; j0 < m.nb; j0 += 32) {
      const int64_t j = j0 + lane;
      const bool set = predicate(m, i, j, lo_i, hi_i);
      const uint32_t ballot = __ballot_sync(0xffffffffu, set);
      if (FILL && set) col_idx[base + __popc(ballot & ((1u << lane) - 1u))] = static_cast<int32_t>(j);
      if (FILL) base += __popc(ballot); else count += __popc(ballot);
    }
  }
  if (!FILL && lane == 0) row_ptr[row + 1] = count;
}

constexpr int kScanThreads = 1024;
constexpr int kScanPer = 4;  // elements per thread per tile

// In-place inclusive scan of row_ptr[1..R] by a single CTA, tile by tile; nnz = total.
__global__ void __launch_bounds__(kScanThreads) mask_scan_kernel(int32_t* row_ptr, int64_t R,
                                                                 int32_t* nnz_out) {
  __shared__ int32_t warp_sums[kScanThreads / 32];
  __shared__ int32_t carry_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry_s = 0;
  __syncthreads();
  int32_t* a = row_ptr + 1;
  for (int64_t t0 = 0; t0 < R; t0 += int64_t(kScanThreads) * kScanPer) {
    int32_t v[kScanPer];
    int32_t local = 0;
#pragma unroll
    for (int e = 0; e < kScanPer; ++e) {
      const int64_t idx = t0 + int64_t(tid) * kScanPer + e;
      v[e] = idx < R ? a[idx] : 0;
      local += v[e];
    }
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int32_t ws = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, ws, o);
        if (lane >= o) ws += t;
      }
      warp_sums[lane] = ws;
    }
    __syncthreads();
    const int32_t carry = carry_s;
    int32_t run = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + incl - local;
#pragma unroll
    for (int e = 0; e < kScanPer; ++e) {
      const int64_t idx = t0 + int64_t(tid) * kScanPer + e;
      run += v[e];
      if (idx < R) a[idx] = run;
    }
    __syncthreads();
    if (tid == kScanThreads - 1) carry_s = carry + warp_sums[31];
    __syncthreads();
  }
  if (tid == 0) *nnz_out = carry_s;
}

}  // namespace

cudaError_t launch_build_mask(const MaskArgs& a, cudaStream_t stream) {
  MaskDev m;
  m.kind = a.kind;
  m.nb = a.n_pad / a.block_size;
  m.rows = int64_t(a.mask_heads) * m.nb;
  m.bs = a.block_size;
  m.n_valid = a.n_valid;
  m.unit = a.unit_tokens > 0 ? a.unit_tokens : 1;
  m.radius = a.radius;
  m.anchors = a.num_anchors;
  m.step = a.step;
  m.group = a.group_blocks > 0 ? a.group_blocks : 1;
  m.frames = (a.n_valid + m.unit - 1) / m.unit;
  m.budget = a.budget_frames;
  m.dense = a.dense;
  const unsigned blocks = unsigned((m.rows + kWarpsPerBlock - 1) / kWarpsPerBlock);
  mask_rows_kernel<false><<<blocks, kWarpsPerBlock * 32, 0, stream>>>(m, a.row_ptr, a.col_idx);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  mask_scan_kernel<<<1, kScanThreads, 0, stream>>>(a.row_ptr, m.rows, a.nnz_out);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  mask_rows_kernel<true><<<blocks, kWarpsPerBlock * 32, 0, stream>>>(m, a.row_ptr, a.col_idx);
  return cudaGetLastError();
}

}  // namespace lva

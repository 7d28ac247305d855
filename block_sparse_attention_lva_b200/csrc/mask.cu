// mask.cu -- block mask -> per-query-block CSR, built on the GPU in three launches:
//   1. count: one warp per CSR row evaluates the mask predicate for 32 key blocks at a time
//      (or 512 bytes of a dense static mask) and reduces with ballot/popc; the count goes
//      to row_ptr[row + 1];
//   2. scan:  one CTA turns the counts into row offsets in place (inclusive scan of
//      row_ptr[1..R]) and writes nnz;
//   3. fill:  the count warp's pass again, writing each set column at its ballot rank.
// Rows come out in (mask head, query block) order with ascending, unique columns, which is
// a pure function of the parameters: the same CSR on every run.
#include <atomic>
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

// In-place inclusive scan of a[0..R) by a single CTA, tile by tile; *total_out = the sum
// (for the CSR: a = row_ptr + 1, total = nnz).
__global__ void __launch_bounds__(kScanThreads) mask_scan_kernel(int32_t* a, int64_t R,
                                                                 int32_t* total_out) {
  __shared__ int32_t warp_sums[kScanThreads / 32];
  __shared__ int32_t carry_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry_s = 0;
  __syncthreads();
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
  if (tid == 0) *total_out = carry_s;
}

constexpr int kScanTile = kScanThreads * kScanPer;   // elements per CTA of the tiled scan

// Tiled scan: every CTA scans its tile of a[0..R) in place (inclusive, local) and
// writes the tile's sum to sums[tile].
__global__ void __launch_bounds__(kScanThreads) scan_tiles_kernel(int32_t* a, int64_t R, int32_t* sums) {
  __shared__ int32_t warp_sums[kScanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t0 = int64_t(blockIdx.x) * kScanTile;
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
  int32_t run = (warp > 0 ? warp_sums[warp - 1] : 0) + incl - local;
#pragma unroll
  for (int e = 0; e < kScanPer; ++e) {
    const int64_t idx = t0 + int64_t(tid) * kScanPer + e;
    run += v[e];
    if (idx < R) a[idx] = run;
  }
  if (tid == kScanThreads - 1) sums[blockIdx.x] = warp_sums[31];
}

// The 16 nonzero-byte flags of a 16-byte vector as 16 bits (bit b = byte b is nonzero).
__device__ __forceinline__ uint32_t nonzero_bits16(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t m = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    // bit 7 of each byte = (byte != 0); the product gathers bits 7, 15, 23, 31 into bits
    // 28..31 (the four partial products land on distinct bit positions: no carries)
    const uint32_t t = (((w[k] & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w[k]) & 0x80808080u;
    m |= ((t * 0x00204081u) >> 28) << (4 * k);
  }
  return m;
}

constexpr int kPackWarps = 8;
// Static masks, pass 1: one warp per row reads the dense row once (16 bytes per lane, eight
// loads in flight) and writes it as bits -- bit j of word j / 32 of the packed row (wpr
// words, the tail words zero) -- and its count to cnt[row].
__global__ void __launch_bounds__(kPackWarps * 32) mask_pack_kernel(const uint8_t* dense, int64_t rows, int64_t nb,
                                                                  int64_t wpr, uint32_t* packed, int32_t* cnt) {
  const int lane = threadIdx.x & 31;
  const bool vec = nb % 16 == 0 && (reinterpret_cast<uintptr_t>(dense) & 15) == 0;
  for (int64_t row = int64_t(blockIdx.x) * kPackWarps + (threadIdx.x >> 5); row < rows;
       row += int64_t(gridDim.x) * kPackWarps) {
    const uint8_t* src = dense + row * nb;
    uint32_t* dst = packed + row * wpr;
    int32_t count = 0;
    if (vec) {
      // up to 4096 columns per round: all of a lane's loads are issued before any is used
      constexpr int kLoads = 8;
      for (int64_t r0 = 0; r0 < nb; r0 += 512 * kLoads) {
        uint4 v[kLoads];
#pragma unroll
        for (int u = 0; u < kLoads; ++u) {
          const int64_t j = r0 + u * 512 + lane * 16;
          v[u] = j < nb ? __ldcs(reinterpret_cast<const uint4*>(src + j)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kLoads; ++u) {
          const int64_t j0 = r0 + u * 512, j = j0 + lane * 16;
          const uint32_t m16 = nonzero_bits16(v[u]);
          count += __popc(m16);
          const uint32_t hi = __shfl_down_sync(0xffffffffu, m16, 1);
          if (!(lane & 1) && j < nb) dst[j0 / 32 + lane / 2] = m16 | (hi << 16);
        }
      }
      count = __reduce_add_sync(0xffffffffu, count);
    } else {
      for (int64_t j0 = 0; j0 < nb; j0 += 32) {
        const int64_t j = j0 + lane;
        const uint32_t b = __ballot_sync(0xffffffffu, j < nb && src[j] != 0);
        if (lane == 0) dst[j0 / 32] = b;
        count += __popc(b);
      }
    }
    for (int64_t w = (nb + 31) / 32 + lane; w < wpr; w += 32) dst[w] = 0;
    if (lane == 0) cnt[row] = count;
  }
}

// Static masks, pass 3: one warp per row.  Its CSR offsets come from the tile-local
// inclusive scan of the counts (cnt) plus the scanned tile sums (sums, absent for a single
// tile); the warp writes row_ptr[row + 1] and expands the packed bits into ascending column
// indices, 1024 columns (one word per lane) at a time.  Each lane writes its word's set bits
// (16-bit offsets from the round's first column, two per step) into a shared-memory run at
// its exclusive prefix count; the run starts `sh` entries in, where sh aligns the run's
// first column index to 16 bytes in col_idx, so that the warp copies it out with 16-byte
// stores (4 indices per lane per step; the run's two ends with plain stores).  The next
// round's words are loaded before this round is expanded.
__global__ void __launch_bounds__(kPackWarps * 32) mask_fill_packed_kernel(const uint32_t* packed, int64_t rows,
                                                                         int64_t nb, int64_t wpr,
                                                                         const int32_t* cnt, const int32_t* sums,
                                                                         int32_t* row_ptr, int32_t* col_idx) {
  __shared__ __align__(16) uint16_t stage[kPackWarps][1024 + 8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint16_t* st = stage[warp];
  for (int64_t row = int64_t(blockIdx.x) * kPackWarps + warp; row < rows; row += int64_t(gridDim.x) * kPackWarps) {
    const int64_t tile = row / kScanTile;
    const int32_t off = (sums != nullptr && tile > 0) ? sums[tile - 1] : 0;
    int32_t base = off + ((row % kScanTile) > 0 ? cnt[row - 1] : 0);
    if (lane == 0) {
      row_ptr[row + 1] = off + cnt[row];
      if (row == 0) row_ptr[0] = 0;
    }
    const uint32_t* src = packed + row * wpr;
    const int nw = int((nb + 31) / 32);
    int32_t* dst = col_idx + base;
    uint32_t next = lane < nw ? __ldcs(src + lane) : 0u;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      uint32_t word = next;
      next = w0 + 32 + lane < nw ? __ldcs(src + w0 + 32 + lane) : 0u;
      const int c = __popc(word);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      const int sh = int((reinterpret_cast<uintptr_t>(dst) >> 2) & 3);
      int pos = incl - c + sh;
      const uint32_t off0 = uint32_t(lane) * 32u;          // the word's first column in the round
      while (word != 0u) {
        const uint32_t rest = word & (word - 1u);
        st[pos] = uint16_t(off0 + uint32_t(__ffs(word) - 1));
        if (rest != 0u) st[pos + 1] = uint16_t(off0 + uint32_t(__ffs(rest) - 1));
        pos += rest != 0u ? 2 : 1;
        word = rest & (rest - 1u);
      }
      __syncwarp();
      const int32_t col0 = w0 * 32;
      const int end = total + sh;                          // run entries [sh, end) -> dst[0 ...]
      for (int c4 = lane * 4; c4 < end; c4 += 128) {
        const uint2 raw = *reinterpret_cast<const uint2*>(st + c4);
        const int32_t v0 = col0 + int32_t(raw.x & 0xffffu), v1 = col0 + int32_t(raw.x >> 16);
        const int32_t v2 = col0 + int32_t(raw.y & 0xffffu), v3 = col0 + int32_t(raw.y >> 16);
        int32_t* o = dst + (c4 - sh);
        if (c4 >= sh && c4 + 4 <= end) {
          *reinterpret_cast<int4*>(o) = make_int4(v0, v1, v2, v3);
        } else {
          if (c4 >= sh && c4 < end) o[0] = v0;
          if (c4 + 1 >= sh && c4 + 1 < end) o[1] = v1;
          if (c4 + 2 >= sh && c4 + 2 < end) o[2] = v2;
          if (c4 + 3 >= sh && c4 + 3 < end) o[3] = v3;
        }
      }
      __syncwarp();
      dst += total;
    }
  }
}

// Scratch of lva_build_block_mask_noalloc: the workspace of the packed static build, held
// in the library's own device memory for callers that cannot allocate any.  Every device
// that loads the library holds the array until the process exits; every call uses all of
// it that it needs, so calls that overlap on the GPU race.  Nothing in it needs to start at
// zero: a build writes each scratch byte it reads earlier in the same build.
constexpr int64_t kNoAllocScratchBytes = int64_t(16) << 20;
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
std::atomic<void*> g_noalloc_ptr[kMaxCachedDevices] = {};

// Device address of the current device's scratch array.  In host code the array's name
// stands for a host-side shadow, not device memory, so the address is looked up (once per
// device, with that device current) and passed to the kernels.
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cacheable = dev >= 0 && dev < kMaxCachedDevices;
  if (cacheable) {
    void* cached = g_noalloc_ptr[dev].load(std::memory_order_acquire);
    if (cached != nullptr) { *out = cached; return cudaSuccess; }
  }
  void* ptr = nullptr;
  e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  if (ptr == nullptr || (reinterpret_cast<uintptr_t>(ptr) & 255) != 0) return cudaErrorInvalidDevicePointer;
  if (cacheable) g_noalloc_ptr[dev].store(ptr, std::memory_order_release);
  *out = ptr;
  return cudaSuccess;
}

}  // namespace

int64_t mask_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Workspace: the packed rows (rows x wpr words), the row counts (rows words, scanned in
// place tile by tile) and the tile sums.
int64_t mask_workspace_bytes(int kind, int64_t rows, int64_t nb) {
  if (kind != kStatic) return 0;
  const int64_t wpr = ((nb + 31) / 32 + 3) / 4 * 4;
  const int64_t tiles = (rows + kScanTile - 1) / kScanTile;
  return rows * wpr * 4 + (rows * 4 + 15) / 16 * 16 + (tiles * 4 + 15) / 16 * 16;
}

cudaError_t launch_build_mask_packed(const MaskArgs& a, void* workspace, cudaStream_t stream) {
  const int64_t nb = a.n_pad / a.block_size;
  const int64_t rows = int64_t(a.mask_heads) * nb;
  const int64_t wpr = ((nb + 31) / 32 + 3) / 4 * 4;
  uint32_t* packed = static_cast<uint32_t*>(workspace);
  int32_t* cnt = reinterpret_cast<int32_t*>(packed + rows * wpr);
  int32_t* sums = cnt + (rows + 3) / 4 * 4;
  const int64_t tiles = (rows + kScanTile - 1) / kScanTile;
  // One warp per row (a grid-stride form with one wave of CTAs measured slower).
  const unsigned pack_blocks = unsigned((rows + kPackWarps - 1) / kPackWarps);
  const unsigned fill_blocks = pack_blocks;
  mask_pack_kernel<<<pack_blocks, kPackWarps * 32, 0, stream>>>(a.dense, rows, nb, wpr, packed, cnt);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (tiles == 1) {
    mask_scan_kernel<<<1, kScanThreads, 0, stream>>>(cnt, rows, a.nnz_out);
  } else {
    scan_tiles_kernel<<<unsigned(tiles), kScanThreads, 0, stream>>>(cnt, rows, sums);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mask_scan_kernel<<<1, kScanThreads, 0, stream>>>(sums, tiles, a.nnz_out);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  mask_fill_packed_kernel<<<fill_blocks, kPackWarps * 32, 0, stream>>>(packed, rows, nb, wpr, cnt,
                                                                  tiles == 1 ? nullptr : sums, a.row_ptr,
                                                                  a.col_idx);
  return cudaGetLastError();
}

cudaError_t launch_build_mask_noalloc(const MaskArgs& a, cudaStream_t stream) {
  const int64_t nb = a.n_pad / a.block_size;
  const int64_t need = mask_workspace_bytes(a.kind, int64_t(a.mask_heads) * nb, nb);
  if (need == 0) return launch_build_mask(a, stream);
  if (need > kNoAllocScratchBytes) return cudaErrorInvalidValue;   // checked by the caller first
  void* scratch = nullptr;
  const cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  return launch_build_mask_packed(a, scratch, stream);
}

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
  mask_scan_kernel<<<1, kScanThreads, 0, stream>>>(a.row_ptr + 1, m.rows, a.nnz_out);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  mask_rows_kernel<true><<<blocks, kWarpsPerBlock * 32, 0, stream>>>(m, a.row_ptr, a.col_idx);
  return cudaGetLastError();
}

}  // namespace lva

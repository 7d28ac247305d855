// calib.cu -- the selection and aggregation steps of static-mask calibration.
//
// CalibAtt page ("Accelerating Text-to-Video Generation with Calibrated Sparse Attention"),
// section 2 A:
//   A.1  for every query block, keep the fewest key blocks whose cumulative energy reaches
//        the threshold eps(t) (select_kernel);
//   A.2  average the per-prompt masks and keep a block when the fraction of calibration
//        prompts that selected it reaches the agreement threshold rho (aggregate_kernel).
//
// The selection decision is an integer taken from floating point, so its arithmetic is
// fixed exactly: energies (float32) in descending order, equal energies by ascending key
// block index; cumulative sums S_k taken one float64 addition at a time in that order; the
// count is the smallest k with S_k >= eps * S_nb (float64 product).  The same decision can
// then be reproduced bit for bit by any IEEE float64 implementation.
#include <cfloat>
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace lva {
namespace {

constexpr int kSelThreads = 256;

// One CTA per energy row (grid-stride): a bitonic sort of 64-bit keys (inverted energy
// bits above the index, so ascending keys = descending energy, then ascending index), one
// thread's sequential float64 prefix sums, the first prefix reaching the target, and the
// 0/1 mask row.  Shared memory: p2 keys + (nb + 1) prefix sums.
__global__ void __launch_bounds__(kSelThreads) select_kernel(const float* __restrict__ energy,
                                                             uint8_t* __restrict__ mask, int64_t rows,
                                                             int nb, int p2, double eps, int* err) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem);
  double* prefix = reinterpret_cast<double*>(smem + size_t(p2) * 8);
  __shared__ int s_bad, s_k;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const float* e = energy + row * nb;
    uint8_t* out = mask + row * nb;
    if (threadIdx.x == 0) { s_bad = 0; s_k = nb; }
    __syncthreads();
    for (int j = threadIdx.x; j < p2; j += kSelThreads) {
      uint64_t key = ~0ull;                                   // padding sorts last
      if (j < nb) {
        float v = e[j] + 0.0f;                                // -0 becomes +0
        if (!(v >= 0.f && v <= FLT_MAX)) { s_bad = 1; v = 0.f; }   // negative, inf or NaN
        key = (uint64_t(~__float_as_uint(v)) << 32) | uint32_t(j);
      }
      keys[j] = key;
    }
    __syncthreads();
    if (s_bad) {
      // An energy that is not a finite non-negative number: the row selects nothing.
      if (threadIdx.x == 0) report_fault(err, 1, int(row & 0x7fffffff));
      for (int j = threadIdx.x; j < nb; j += kSelThreads) out[j] = 0;
      __syncthreads();
      continue;
    }
    for (int k = 2; k <= p2; k <<= 1) {
      for (int jj = k >> 1; jj > 0; jj >>= 1) {
        for (int x = threadIdx.x; x < p2; x += kSelThreads) {
          const int y = x ^ jj;
          if (y > x) {
            const uint64_t a = keys[x], b = keys[y];
            if ((a > b) == ((x & k) == 0)) { keys[x] = b; keys[y] = a; }
          }
        }
        __syncthreads();
      }
    }
    if (threadIdx.x == 0) {
      double acc = 0.0;
      prefix[0] = 0.0;
      for (int m = 0; m < nb; ++m) {
        acc = acc + double(__uint_as_float(~uint32_t(keys[m] >> 32)));
        prefix[m + 1] = acc;
      }
    }
    __syncthreads();
    // Prefix sums of non-negative terms never decrease, so each thread's first hit in its
    // strided walk is its smallest; the CTA takes the minimum.  S_nb >= eps * S_nb for
    // eps <= 1, so some m always qualifies.
    const double target = eps * prefix[nb];
    for (int m = threadIdx.x; m <= nb; m += kSelThreads) {
      if (prefix[m] >= target) { atomicMin(&s_k, m); break; }
    }
    __syncthreads();
    const int kc = s_k;
    for (int m = threadIdx.x; m < nb; m += kSelThreads)
      out[uint32_t(keys[m])] = m < kc ? 1 : 0;
    __syncthreads();   // shared memory is reused by the next row
  }
}

__global__ void aggregate_kernel(const uint8_t* __restrict__ masks, uint8_t* __restrict__ out,
                                 int prompts, int64_t count, double threshold) {
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t x = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; x < count; x += stride) {
    int c = 0;
    for (int p = 0; p < prompts; ++p) c += masks[int64_t(p) * count + x] != 0;
    out[x] = double(c) >= threshold ? 1 : 0;
  }
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  int p2 = 1;
  while (p2 < a.nb) p2 <<= 1;
  const size_t smem = size_t(p2) * 8 + size_t(a.nb + 1) * 8;
  static DeviceFlags attr_set = {};
  cudaError_t e = once_per_device(attr_set, [] {
    const int max_smem = (kSelectMaxBlocks + kSelectMaxBlocks + 1) * 8;
    return cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
  });
  if (e != cudaSuccess) return e;
  const int64_t grid = a.rows < int64_t(sm_count()) * 8 ? a.rows : int64_t(sm_count()) * 8;
  select_kernel<<<unsigned(grid), kSelThreads, smem, stream>>>(a.energy, a.mask, a.rows, a.nb, p2,
                                                               a.eps, a.err);
  return cudaGetLastError();
}

cudaError_t launch_aggregate(const AggregateArgs& a, cudaStream_t stream) {
  if (a.count == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (a.count + threads - 1) / threads;
  const int64_t cap = int64_t(sm_count()) * 16;
  if (blocks > cap) blocks = cap;
  aggregate_kernel<<<unsigned(blocks), threads, 0, stream>>>(a.masks, a.out, a.prompts, a.count,
                                                              a.threshold);
  return cudaGetLastError();
}

}  // namespace lva

// selftest.cu -- exercises the bounded mbarrier wait that every pipeline kernel here uses.
//
// One CTA of two warps.  Lane 0 of warp 0 waits on a freshly initialised mbarrier through
// mbar_wait (ptx.cuh), exactly as the attention and energy pipelines wait on their hand-offs;
// warp 1 plays the other role:
//   mode 0: nothing ever arrives, so the wait runs to its kWaitLimitNs limit;
//   mode 1: warp 1 raises the CTA's abort flag after about 1 ms, so the wait gives up early;
//   mode 2: warp 1 arrives on the barrier after about 1 ms, so the wait completes.
// A wait that gives up records LVA_ERR_TIMEOUT (5) in the device error word with detail
// 100 + mode, as the pipelines do; a completed wait records nothing.  Every loop here is
// bounded by %globaltimer, so no mode can hang the GPU.
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace lva {
namespace {

constexpr unsigned long long kPeerDelayNs = 1000000ull;  // 1 ms

__global__ void __launch_bounds__(64) wait_selftest_kernel(int mode, int* err) {
  __shared__ alignas(8) uint64_t bar;
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  const int warp = int(threadIdx.x / 32), lane = int(threadIdx.x % 32);
  if (warp == 0 && lane == 0) {
    if (!mbar_wait(b, 0, abort_flag)) report_fault(err, 5, 100 + mode);
  } else if (warp == 1 && lane == 0 && mode != 0) {
    const unsigned long long t0 = global_timer_ns();
    while (global_timer_ns() - t0 < kPeerDelayNs) {
    }
    if (mode == 1) {
      *abort_flag = 1;
    } else {
      mbar_arrive(b);
    }
  }
}

}  // namespace

cudaError_t launch_wait_selftest(int mode, int* err, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 64, 0, stream>>>(mode, err);
  return cudaGetLastError();
}

}  // namespace lva

// broadcast.cu -- copy the output of anchor query blocks to the blocks that repeat them.
//
// For heads whose spatial rows repeat (the CalibAtt page, "Accelerating Text-to-Video
// Generation with Calibrated Sparse Attention", section 2 A.3 and B), attention runs only on
// anchor blocks and this kernel replicates their O rows and LSE to the other blocks.  One CTA
// per (plane, query block); blocks whose source is themselves exit at once.  HBM-bound:
// 2 * Bs * (d * 2 + 4) bytes moved per repeated block.
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace lva {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) broadcast_kernel(uint8_t* __restrict__ o, float* __restrict__ lse,
                                                             int H, int64_t nb, int bs, int row_bytes,
                                                             const int32_t* __restrict__ src_map,
                                                             int src_heads, int* err) {
  const int64_t item = blockIdx.x;
  const int64_t plane = item / nb;
  const int64_t i = item - plane * nb;
  const int64_t map_row = int64_t(src_heads == 1 ? 0 : int(plane % H)) * nb;
  const int32_t src = __ldg(src_map + map_row + i);
  if (src == i) return;
  if (src < 0 || src >= nb || __ldg(src_map + map_row + src) != src) {
    if (threadIdx.x == 0) report_fault(err, 1, int((map_row + i) & 0x7fffffff));
    return;
  }
  const int64_t plane_rows = nb * bs;
  const uint4* s = reinterpret_cast<const uint4*>(o + (plane * plane_rows + int64_t(src) * bs) * row_bytes);
  uint4* d = reinterpret_cast<uint4*>(o + (plane * plane_rows + i * bs) * row_bytes);
  const int n16 = bs * row_bytes / 16;
  for (int k = threadIdx.x; k < n16; k += kThreads) d[k] = s[k];
  for (int r = threadIdx.x; r < bs; r += kThreads)
    lse[plane * plane_rows + i * bs + r] = lse[plane * plane_rows + int64_t(src) * bs + r];
}

}  // namespace

cudaError_t launch_broadcast(const BroadcastArgs& a, cudaStream_t stream) {
  const int64_t nb = a.n_pad / a.block_size;
  const int64_t items = int64_t(a.B) * a.H * nb;
  if (items == 0) return cudaSuccess;
  broadcast_kernel<<<dim3(unsigned(items)), kThreads, 0, stream>>>(
      static_cast<uint8_t*>(a.o), a.lse, a.H, nb, a.block_size, a.d * 2, a.query_src, a.src_heads, a.err);
  return cudaGetLastError();
}

}  // namespace lva

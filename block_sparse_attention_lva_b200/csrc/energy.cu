// energy.cu -- block energies of softmax attention for sm_100a (TMA + tcgen05 + TMEM).
//
// CalibAtt page ("Accelerating Text-to-Video Generation with Calibrated Sparse Attention"),
// section 2 A.1: during offline calibration the attention matrix is cut into Bs x Bs
// blocks and, for every query block i, the energy toward key block j is the sum of its
// attention scores.  Here
//
//   E[b,h,i,j] = sum over real rows r of block i and real keys c of block j of
//                exp(scale * <q_r, k_c> - LSE_r),
//
// with LSE_r the row log-sum-exp over all real keys (natural log, scale included) -- the
// LSE that the attention call returns with the all-ones mask.  One CTA computes one
// (b, h, i) over the key blocks of its CSR row (all of them for a dense calibration pass)
// and writes the whole energy row: listed blocks get their energy, the others 0.
//
// Warp roles (320 threads, up to two CTAs per SM):
//   warp 0       TMA producer: Q tile once, then K_j tiles into a 2-slot ring;
//   warp 1       MMA issuer (one thread): S_b = Q K_j^T into one of two TMEM buffers;
//   warps 2..9   reduction: thread = (query row, column half), exactly as in the attention
//                kernel's softmax; the warp sums its 32 x BN/2 probabilities with a fixed
//                shuffle tree, and the eight warp sums of a block are added in warp order,
//                so the result does not depend on timing.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace lva {
namespace {

constexpr int EBM = 128;            // query rows per MMA tile (TMEM lanes)
constexpr int kRedWarp0 = 2;
constexpr int kRedWarps = 8;
constexpr int kEThreads = 32 * (kRedWarp0 + kRedWarps);
constexpr int kChunk = 256;         // list positions buffered before the warp sums are combined
constexpr uint32_t kETmemCols = 256;

struct EnergyParams {
  int H, nb, mask_heads;
  int64_t n_pad, n_valid;
  float scale_log2;                 // scale * log2(e)
  const float* lse;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int64_t col_len;
  float* energy;                    // [B, H, nb, nb]
  int* err;
};

template <int D, int BN>
struct ECfg {
  static constexpr int KST = 2;
  static constexpr int Q_BYTES = EBM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_BAR = OFF_K + KST * KV_BYTES;
  // barriers: q_full, k_full[KST], k_empty[KST], s_full[2], s_free[2], final, group[2]
  static constexpr int B_Q = 0, B_KF = 1, B_KE = B_KF + KST, B_SF = B_KE + KST, B_SE = B_SF + 2,
                       B_FIN = B_SE + 2, B_GRP = B_FIN + 1, NUM_BARS = B_GRP + 2;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_RED = (OFF_MISC + 16 + 15) / 16 * 16;   // [kChunk][kRedWarps] floats
  static constexpr int SMEM_BYTES = OFF_RED + kChunk * kRedWarps * 4;
  static_assert(2 * SMEM_BYTES <= 227 * 1024, "two CTAs per SM");
  static_assert(D <= 128 && BN <= 128, "TMEM layout");
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(EBM, BN, 0, 0);
};

template <int D, int BN>
__global__ void __launch_bounds__(kEThreads, 2) block_energy_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const EnergyParams p) {
  using C = ECfg<D, BN>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t s_base = smem_u32(smem);
  if (s_base & 1023u) {
    if (threadIdx.x == 0) report_fault(p.err, 4, 1023);
    return;
  }
  const uint32_t sQ = s_base + C::OFF_Q, sK = s_base + C::OFF_K;
  const uint32_t bar0 = s_base + C::OFF_BAR;
  const uint32_t bar_q = bar0 + 8u * C::B_Q;
  auto bar_k_full = [&](int s) { return bar0 + 8u * (C::B_KF + s); };
  auto bar_k_empty = [&](int s) { return bar0 + 8u * (C::B_KE + s); };
  auto bar_s_full = [&](int b) { return bar0 + 8u * (C::B_SF + b); };
  auto bar_s_free = [&](int b) { return bar0 + 8u * (C::B_SE + b); };
  const uint32_t bar_final = bar0 + 8u * C::B_FIN;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  volatile int* never = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int64_t item = blockIdx.x;
  const int64_t plane = item / p.nb;
  const int i = int(item - plane * p.nb);
  const int h = int(plane % p.H);
  const int64_t csr = int64_t(p.mask_heads == 1 ? 0 : h) * p.nb + i;
  // CSR row, validated by every warp from the same memory (same answer everywhere).
  const int32_t a = __ldg(p.row_ptr + csr), b_end = __ldg(p.row_ptr + csr + 1);
  bool bad = !(a >= 0 && b_end >= a && int64_t(b_end) <= p.col_len);
  if (!bad) {
    bool lane_bad = false;
    for (int32_t t = a + lane; t < b_end; t += 32) {
      const int32_t j = __ldg(p.col_idx + t);
      const int32_t prev = t > a ? __ldg(p.col_idx + t - 1) : -1;
      lane_bad |= (j < 0 || j >= p.nb || j <= prev);   // in range, strictly ascending
    }
    bad = __any_sync(0xffffffffu, lane_bad);
  }
  const int32_t start = bad ? 0 : a;
  const int n = bad ? 0 : b_end - a;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::KST; ++s) { mbar_init(bar_k_full(s), 1); mbar_init(bar_k_empty(s), 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_s_full(b), 1);
      mbar_init(bar_s_free(b), kRedWarps);
      mbar_init(bar0 + 8u * (C::B_GRP + b), kRedWarps);
    }
    mbar_init(bar_final, 1);
    *abort_flag = 0;
    *never = 0;
    mbar_fence_init();
  }
  if (warp == 1) { tmem_alloc(smem_u32(tmem_slot), kETmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer: Q, K
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k);
      const int32_t q_row = int32_t(plane * p.n_pad + int64_t(i) * BN);
      mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
      for (int c = 0; c < D / 64; ++c) tma_load_2d(sQ + c * EBM * 128, &tm_q, c * 64, q_row, bar_q);
      int issued = 0;
      for (int t = 0; t < n; ++t) {
        const int s = t % C::KST;
        if (t >= C::KST && !mbar_wait(bar_k_empty(s), ((t / C::KST) - 1) & 1, abort_flag)) {
          *abort_flag = 1; report_fault(p.err, 5, 11); break;
        }
        const int32_t j = __ldg(p.col_idx + start + t);
        const int32_t kv_row = int32_t(plane * p.n_pad + int64_t(j) * BN);
        mbar_arrive_expect_tx(bar_k_full(s), C::KV_BYTES);
        for (int c = 0; c < D / 64; ++c)
          tma_load_2d(sK + s * C::KV_BYTES + c * BN * 128, &tm_k, c * 64, kv_row, bar_k_full(s));
        issued = t + 1;
      }
      if (*abort_flag) {
        // every load issued lands before the CTA exits
        for (int t = (issued > C::KST ? issued - C::KST : 0); t < issued; ++t)
          mbar_wait(bar_k_full(t % C::KST), (t / C::KST) & 1, never);
        mbar_wait(bar_q, 0, never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      const uint64_t q_desc = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t k_desc = smem_desc_sw128(sK, 16, 1024);
      bool ok = mbar_wait(bar_q, 0, abort_flag);
      bool any_mma = false;
      for (int t = 0; ok && t < n; ++t) {
        const int s = t % C::KST, b = t & 1;
        if (!mbar_wait(bar_k_full(s), (t / C::KST) & 1, abort_flag)) { ok = false; break; }
        if (t >= 2 && !mbar_wait(bar_s_free(b), ((t >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint64_t ks = k_desc + uint64_t((s * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_f16_ss(tmem + 128 * b, q_desc + uint64_t(((kk / 4) * EBM * 128 + (kk % 4) * 32) >> 4),
                      ks + uint64_t(((kk / 4) * BN * 128 + (kk % 4) * 32) >> 4), C::IDESC_QK,
                      kk > 0 ? 1u : 0u);
        umma_commit(bar_s_full(b));
        umma_commit(bar_k_empty(s));
        any_mma = true;
      }
      if (!ok) { *abort_flag = 1; report_fault(p.err, 5, 12); }
      if (any_mma) {
        umma_commit(bar_final);
        mbar_wait(bar_final, 0, never);
      }
    }
  } else {
    // ------------------------------------------------------------ reduction warps
    constexpr int HALF = BN / 2;
    const int wid = warp - kRedWarp0;             // 0..7, the fixed order of the warp sums
    const int hf = wid >> 2;                      // column half
    const int sub = warp & 3;                     // TMEM lane quarter this warp may access
    const int row = sub * 32 + lane;
    const uint32_t lane_off = uint32_t(sub * 32) << 16;
    const int64_t grow = int64_t(i) * BN + row;
    float lse2 = 0.f;
    bool row_ok = row < BN && grow < p.n_valid;
    if (row_ok) {
      const float l = __ldg(p.lse + plane * p.n_pad + grow);
      row_ok = (l == l) && l > -INFINITY && l < INFINITY;
      lse2 = row_ok ? l * 1.4426950408889634f : 0.f;
    }
    const float c = p.scale_log2;
    float* erow = p.energy + (plane * p.nb + i) * int64_t(p.nb);
    // Barrier over the eight reduction warps: sync number `seq` uses slot seq & 1; a warp
    // can only arrive for seq + 2 after every warp has arrived for seq + 1, i.e. after all
    // have left the wait for seq, so a slot never runs a phase ahead.  Bounded like every
    // wait here: on a timeout the warp stops instead of blocking the others.
    int seq = 0;
    auto group_sync = [&]() -> bool {
      const uint32_t bar = bar0 + 8u * (C::B_GRP + (seq & 1));
      const uint32_t parity = (seq >> 1) & 1;
      ++seq;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    if (bad && wid == 0 && lane == 0) report_fault(p.err, 1, int(csr & 0x7fffffff));
    // The whole row starts at zero; the sync orders these stores before the sums below.
    for (int j = wid * 32 + lane; j < p.nb; j += kRedWarps * 32) erow[j] = 0.f;
    bool ok = group_sync();
    int flushed = 0;
    for (int t = 0; ok && t < n; ++t) {
      const int b = t & 1;
      const int32_t j = __ldg(p.col_idx + start + t);
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full(b), (t >> 1) & 1, abort_flag))) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[HALF];
#pragma unroll
      for (int q = 0; q < HALF / 32; ++q)
        tmem_ld32(tmem + lane_off + 128 * b + hf * HALF + q * 32,
                  *reinterpret_cast<uint32_t(*)[32]>(sr + q * 32));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_s_free(b));

      // Real keys of this half (only the block holding the sequence end is partial).
      const int64_t valid = p.n_valid - int64_t(j) * BN - hf * HALF;
      float sum = 0.f;
      if (row_ok && valid >= HALF) {
        const uint64_t c2 = f2_pack(c, c), nl2 = f2_pack(-lse2, -lse2);
        uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
        for (int e = 0; e < HALF / 2; ++e) {
          const uint64_t x2 = f2_fma(f2_pack_bits(sr[2 * e], sr[2 * e + 1]), c2, nl2);
          uint64_t p2;
          if (e % 3 == 2) {
            p2 = exp2_poly_f2(x2);
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
          }
          acc[e & 1] = f2_add(acc[e & 1], p2);
        }
        const uint64_t s2 = f2_add(acc[0], acc[1]);
        float s0, s1;
        f2_unpack(s2, s0, s1);
        sum = s0 + s1;
      } else if (row_ok && valid > 0) {
#pragma unroll
        for (int e = 0; e < HALF; ++e)
          if (e < valid) sum += ex2_approx(fmaf(__uint_as_float(sr[e]), c, -lse2));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) red[(t - flushed) * kRedWarps + wid] = sum;

      if (t - flushed == kChunk - 1 || t == n - 1) {
        // Combine the warp sums of the buffered positions, in warp order.
        if (!group_sync()) { ok = false; break; }
        const int cnt = t - flushed + 1;
        for (int x = wid * 32 + lane; x < cnt; x += kRedWarps * 32) {
          float e = 0.f;
#pragma unroll
          for (int w = 0; w < kRedWarps; ++w) e += red[x * kRedWarps + w];
          erow[__ldg(p.col_idx + start + flushed + x)] = e;
        }
        if (!group_sync()) { ok = false; break; }
        flushed = t + 1;
      }
    }
    if (!ok) {
      *abort_flag = 1;
      if (wid == 0 && lane == 0) report_fault(p.err, 5, 13);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kETmemCols);
  }
}

template <int D, int BN>
cudaError_t launch_energy_cfg(const EnergyArgs& a, cudaStream_t stream, const char** why) {
  using C = ECfg<D, BN>;
  const int64_t rows = int64_t(a.B) * a.H * a.n_pad;
  CUtensorMap tq, tk;
  if (!make_rows_map(&tq, a.q, rows, D, EBM) || !make_rows_map(&tk, a.k, rows, D, BN)) {
    *why = "cuTensorMapEncodeTiled failed or is unavailable";
    return cudaErrorInvalidValue;
  }
  static DeviceFlags attr_set = {};
  cudaError_t e = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(block_energy_kernel<D, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::SMEM_BYTES);
  });
  if (e != cudaSuccess) { *why = "cudaFuncSetAttribute(max dynamic smem) failed"; return e; }
  EnergyParams p;
  p.H = a.H;
  p.nb = int(a.n_pad / a.block_size);
  p.mask_heads = a.mask_heads;
  p.n_pad = a.n_pad;
  p.n_valid = a.n_valid;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.lse = a.lse;
  p.row_ptr = a.row_ptr;
  p.col_idx = a.col_idx;
  p.col_len = a.col_len;
  p.energy = a.energy;
  p.err = a.err;
  const int64_t items = rows / a.block_size;
  if (items == 0) return cudaSuccess;
  block_energy_kernel<D, BN><<<dim3(unsigned(items)), kEThreads, C::SMEM_BYTES, stream>>>(tq, tk, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_energy(const EnergyArgs& a, cudaStream_t stream, const char** why) {
  if (a.d == 128 && a.block_size == 128) return launch_energy_cfg<128, 128>(a, stream, why);
  if (a.d == 128 && a.block_size == 64) return launch_energy_cfg<128, 64>(a, stream, why);
  if (a.d == 64 && a.block_size == 128) return launch_energy_cfg<64, 128>(a, stream, why);
  if (a.d == 64 && a.block_size == 64) return launch_energy_cfg<64, 64>(a, stream, why);
  *why = "unsupported (d, block_size)";
  return cudaErrorInvalidValue;
}

}  // namespace lva

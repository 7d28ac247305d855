// attn.cu -- block-sparse FlashAttention-style forward for sm_100a (TMA + tcgen05 + TMEM).
//
// A CTA computes a run of consecutive (batch, head, query block i) items -- one, or 4 or 8
// when the CSR rows are short -- and for each walks only the key blocks listed in CSR row
// (h_m, i): the precomputed skip list of the CalibAtt page ("Accelerating Text-to-Video
// Generation with Calibrated Sparse Attention", section 2 B) or the LVSA window + anchor set
// ("LVSA: Training-Free Sparse Attention for Long Video Diffusion", technical summary
// section 2), with an online softmax, so the cost is proportional to the number of listed
// blocks.  O goes to tile order, or straight to raster order (the inverse token reorder
// fused into the epilogue); Q/K/V rows come from plane-major 2D tensor maps, or from 3D
// maps that gather the window-transposed order in place (the SQuad page's global pass).
//
// Pipeline: three S buffers in TMEM (S_0, S_1, S_2, O = 512 columns).  The softmax writes
// P(t) as bf16 over the first columns of S(t), which O += P(t) V_t then reads, so buffer
// t mod 3 is free again once that P V has completed.  The MMA issuer computes S(t+3) =
// Q K_{t+3}^T then, O += P(t) V_t runs while the softmax works on block t+1, and the softmax
// never waits for a P buffer: it is the only serial chain.  (The LSE-only form has neither P
// nor O: four S buffers, released as soon as the softmax has read them.)
//
// Warp roles (384 threads):
//   warp 0       TMA producer: Q tile once, then K_j tiles into a 3-slot ring;
//   warp 10      TMA producer: V_j tiles into a 3-slot ring;
//   warp 1       MMA issuer (one thread): S_b = Q K_j^T; owns TMEM;
//   warp 11      MMA issuer (one thread): O += P_b V_j (P_b read from TMEM, over S_b);
//   warps 2..9   softmax + epilogue: each warp owns 16 rows of the 128-row tile; lane t and
//                lane t + 16 hold the left and right column halves of one row (the .16x32bx2
//                TMEM shapes), so row maxima and sums meet through one shuffle; O is
//                rescaled in TMEM only when the running max grows by more than 2^8.
//
// The LSE-only form (lva_block_sparse_lse) runs the same roles without the V producer, the
// P V issuer, the P stores and the O epilogue: its softmax only sums.
//
// Shared-memory operands use the 128-byte swizzle that TMA writes: a 64-element (128 B)
// slice of each row, eight rows per 1024-byte atom.  Q and K are K-major; V is read
// MN-major straight from its [keys, d] layout; P is the TMEM A operand of P*V.
#include <cstdint>
#include <type_traits>
#include <cuda.h>
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"
#include "tile_order.cuh"

namespace lva {
namespace {

constexpr int BM = 128;            // query rows per MMA tile (TMEM lanes)
constexpr int kSoftmaxWarp0 = 2;
constexpr int kSoftmaxWarps = 8;   // two warps per TMEM lane quarter: 16 rows each
constexpr int kVWarp = kSoftmaxWarp0 + kSoftmaxWarps;   // V producer, after the softmax warps
constexpr int kPVWarp = kVWarp + 1;                       // issuer of O += P V
constexpr int kThreads = 32 * (kPVWarp + 1);
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when max grows > 2^8
constexpr uint32_t kTmemCols = 512;

// Exponential pairs on the FMA-pipe polynomial: one in four with P packing and stores (of
// 1/2, 1/3, 1/4 and none, 1/4 to 3/8 measured fastest), one in three for the LSE-only form,
// whose FMA pipe has no P work (3.90 ms against 4.09 ms for one in four, 4.32 for one in two).
template <bool LSE_ONLY>
__device__ __forceinline__ constexpr bool kPolyPair(int e) { return LSE_ONLY ? (e % 3 == 2) : (e % 4 == 3); }

struct AttnParams {
  int H, nb, mask_heads;
  int64_t n_pad, n_valid;
  float scale_log2;                // scale * log2(e)
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int64_t col_len;
  __nv_bfloat16* o;                // tile order [planes, n_pad, D], or
  __nv_bfloat16* o_raster;         // when set: raster order [planes, n_valid, D] (o unused)
  Grid3 grid;                      // latent grid and tile of the raster order
  int64_t items;                   // (plane, query block) work items: planes * nb
  int o_align32;                   // O rows start on 32-byte boundaries: 32-byte stores
  int gather_windows;              // 0: rows are plane-major [planes, n_pad, D]; m > 0: q, k,
                                   // v hold m windows per plane and row k of the
                                   // window-transposed order is read through a 3D map
  float* lse;
  const int32_t* query_src;        // NULL or [src_heads, nb]: blocks copied from an anchor
  int src_heads;
  int* err;
};

template <int D, int BN, bool LSE_ONLY>
struct Cfg {
  static constexpr int KST = 3, VST = LSE_ONLY ? 0 : 3;
  // S buffers in TMEM.  With P V, P(t) is written over S(t)'s first columns, so a buffer is
  // free again once O += P(t) V has completed, and three buffers fit next to O.  The
  // LSE-only form has neither P nor O: four buffers, each released as soon as the softmax
  // has read it (3.76 ms against 3.81 ms with two, dense small workload).
  static constexpr int NSB = LSE_ONLY ? 4 : 3;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VST * KV_BYTES;
  // barriers: q_full, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[NSB],
  // s_free[NSB] (LSE only: S read), p_full[NSB] (P stored over S), o_done[NSB] (P*V done:
  // the S buffer is free again), final (Q K^T), final (P V), q_empty (an item's Q K^T done:
  // Q may be replaced), o_free (an item's O read: P V may start the next item)
  static constexpr int B_Q = 0, B_KF = 1, B_KE = B_KF + KST, B_VF = B_KE + KST, B_VE = B_VF + VST,
                       B_SF = B_VE + VST, B_SE = B_SF + NSB, B_P = B_SE + NSB, B_O = B_P + NSB,
                       B_FIN = B_O + NSB, B_FIN_PV = B_FIN + 1, B_QE = B_FIN_PV + 1, B_OF = B_QE + 1,
                       NUM_BARS = B_OF + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  // At least 120 KB so that one CTA (and one 512-column TMEM allocation) is resident per SM.
  static constexpr int SMEM_RAW = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = SMEM_RAW > 120 * 1024 ? SMEM_RAW : 120 * 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  // TMEM columns: S_b at 128 b (P_b, bf16 pairs, over its first 64 columns), O at 384 (the
  // LSE-only form has no O: its fourth S buffer is there)
  static constexpr uint32_t TM_S = 0, TM_O = 384;
  static_assert(D <= 128 && BN <= 128, "TMEM layout");
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, 0, 1);
};

// The CSR row of a work item, checked so that no read or TMA coordinate leaves its buffer
// and so that no key block is counted twice: the row must lie inside col_len and list
// strictly ascending block indices in [0, nb).  Called by every thread (whole warps); each
// warp checks the row cooperatively, so every role reaches the same answer from the same
// memory.
__device__ __forceinline__ int csr_row(const AttnParams& p, int64_t row, int32_t& start,
                                       bool& bad) {
  const int32_t a = __ldg(p.row_ptr + row), b = __ldg(p.row_ptr + row + 1);
  bad = !(a >= 0 && b >= a && int64_t(b) <= p.col_len);
  start = 0;
  if (bad) return 0;
  bool lane_bad = false;
  for (int32_t t = a + int32_t(threadIdx.x & 31); t < b; t += 32) {
    const int32_t j = __ldg(p.col_idx + t);
    const int32_t prev = t > a ? __ldg(p.col_idx + t - 1) : -1;
    lane_bad |= (j < 0 || j >= p.nb || j <= prev);
  }
  bad = __any_sync(0xffffffffu, lane_bad);
  if (bad) return 0;
  start = a;
  return b - a;
}

// O *= alpha for this thread's half row (the lazy rescale, rare once an item's running max
// has settled), out of line so that its code and registers stay out of the softmax loop.
template <int DH>
__device__ __noinline__ void rescale_o(uint32_t taddr, float alpha) {
#pragma unroll 1
  for (int q = 0; q < DH / 32; ++q) {
    uint32_t ov[32];
    tmem_ld_16x2_32<DH>(taddr + q * 32, ov);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
    tmem_st_16x2_32<DH>(taddr + q * 32, ov);
  }
}

// NEG: the softmax scale is negative, so the row max of scale * s is scale * min(s) (a
// separate instantiation keeps the positive-scale loop free of that path).
template <int D, int BN, int KPC, bool LSE_ONLY, bool NEG>
__global__ void __launch_bounds__(kThreads, 1) bsa_fwd_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = Cfg<D, BN, LSE_ONLY>;
  // 128-byte-swizzled TMA tiles need 1024-byte aligned shared memory.
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t s_base = smem_u32(smem);
  if (s_base & 1023u) {                           // never expected; checked rather than assumed
    if (threadIdx.x == 0) report_fault(p.err, 4, 1023);
    return;
  }
  const uint32_t sQ = s_base + C::OFF_Q, sK = s_base + C::OFF_K, sV = s_base + C::OFF_V;
  const uint32_t bar0 = s_base + C::OFF_BAR;
  const uint32_t bar_q = bar0 + 8u * C::B_Q;
  auto bar_k_full = [&](int s) { return bar0 + 8u * (C::B_KF + s); };
  auto bar_k_empty = [&](int s) { return bar0 + 8u * (C::B_KE + s); };
  auto bar_v_full = [&](int s) { return bar0 + 8u * (C::B_VF + s); };
  auto bar_v_empty = [&](int s) { return bar0 + 8u * (C::B_VE + s); };
  auto bar_s_full = [&](int b) { return bar0 + 8u * (C::B_SF + b); };
  auto bar_s_free = [&](int b) { return bar0 + 8u * (C::B_SE + b); };
  auto bar_p_full = [&](int b) { return bar0 + 8u * (C::B_P + b); };
  auto bar_o_done = [&](int b) { return bar0 + 8u * (C::B_O + b); };
  const uint32_t bar_final = bar0 + 8u * C::B_FIN;
  const uint32_t bar_final_pv = bar0 + 8u * C::B_FIN_PV;
  const uint32_t bar_q_empty = bar0 + 8u * C::B_QE;
  const uint32_t bar_o_free = bar0 + 8u * C::B_OF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  // Stays zero: the drain waits after an abort are bounded by time alone.
  volatile int* never = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work items: (plane, query block), plane-major with the query block fastest.  The CTA
  // takes a run of consecutive items (below).  Every role walks the same items; pipeline
  // positions T count key blocks over all items of this CTA, so ring slots, S buffers and
  // their barrier phases simply continue from one item to the next, and the next item's Q
  // load and first Q K^T overlap the current item's epilogue.
  const int items = int(p.items);               // < 2^31: B*H*n_pad < 2^31 is enforced
  // This CTA's items: a run of consecutive query blocks (same plane, overlapping key lists,
  // so their K/V tiles stay in L2); CTAs are launched in item order.
  const int it_begin = int(blockIdx.x) * KPC;
  const int it_end = it_begin + KPC < items ? it_begin + KPC : items;
  // Per item: whether it is computed here, its CSR row start and length (every warp derives
  // the same values from the same memory; a corrupt row counts as empty).
  struct Item { int plane; int i; int32_t start; int n; bool skip; bool bad; };
  auto item_at = [&](int it) -> Item {
    Item r;
    r.plane = it / p.nb;
    r.i = it - r.plane * p.nb;
    const int h = r.plane % p.H;
    r.skip = p.query_src != nullptr &&
             __ldg(p.query_src + int64_t(p.src_heads == 1 ? 0 : h) * p.nb + r.i) != r.i;
    r.n = 0; r.start = 0; r.bad = false;
    if (!r.skip) r.n = csr_row(p, int64_t(p.mask_heads == 1 ? 0 : h) * p.nb + r.i, r.start, r.bad);
    return r;
  };

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_q_empty, 1);
    for (int s = 0; s < C::KST; ++s) { mbar_init(bar_k_full(s), 1); mbar_init(bar_k_empty(s), 1); }
    for (int s = 0; s < C::VST; ++s) { mbar_init(bar_v_full(s), 1); mbar_init(bar_v_empty(s), 1); }
    for (int b = 0; b < C::NSB; ++b) {
      mbar_init(bar_s_full(b), 1);
      mbar_init(bar_s_free(b), kSoftmaxWarps);
      mbar_init(bar_p_full(b), kSoftmaxWarps);
      mbar_init(bar_o_done(b), 1);
    }
    mbar_init(bar_o_free, kSoftmaxWarps);
    mbar_init(bar_final, 1);
    mbar_init(bar_final_pv, 1);
    *abort_flag = 0;
    *never = 0;
    mbar_fence_init();
  }
  if (warp == 1) { tmem_alloc(smem_u32(tmem_slot), kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // TMA load of the 64-element column chunk c of the rows [k0, k0 + box) of a plane:
  // plane-major rows, or (window-gather maps) row k = pos * m + a of the window-transposed
  // order, which is row a * w + pos of the input: coordinates (c * 64, pos, plane * m + a).
  auto load_rows = [&](uint32_t dst, const void* tmap, int c, int64_t plane, int64_t k0, uint32_t bar) {
    if (p.gather_windows == 0) {
      tma_load_2d(dst, tmap, c * 64, int32_t(plane * p.n_pad + k0), bar);
    } else {
      const int64_t m = p.gather_windows;
      const int64_t pos = k0 / m;
      tma_load_3d(dst, tmap, c * 64, int32_t(pos), int32_t(plane * m + (k0 - pos * m)), bar);
    }
  };

  // The producer and issuer warps wait in mbarrier.try_wait (the warp sleeps until the phase
  // completes), so their waits take no issue slots from the softmax warps that share their
  // schedulers; the softmax warps poll, since their hand-offs are on the critical path.
  //
  // A TMA producer: key block T (over all items) goes to slot T % ST of a ring whose slots
  // are released by `empty` barriers; after an abort it waits for the loads still in flight.
  auto produce = [&](const void* tmap, uint32_t ring, int ST, uint32_t full0, uint32_t empty0, int code,
                     bool with_q) {
    uint32_t T = 0;         // key blocks issued so far
    int nq = 0;             // Q tiles issued so far
    for (int it = it_begin; it < it_end; ++it) {
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;     // one decision for the warp
      const Item w = item_at(it);
      if (w.n == 0) continue;
      if (lane == 0) {
        if (with_q) {
          // Q is single-buffered: the previous item's Q K^T must have completed.
          if (nq > 0 && !mbar_wait_sleep(bar_q_empty, (nq - 1) & 1, abort_flag)) {
            *abort_flag = 1; report_fault(p.err, 5, 8);
          } else {
            mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
            for (int c = 0; c < D / 64; ++c)
              load_rows(sQ + c * BM * 128, &tm_q, c, w.plane, int64_t(w.i) * BN, bar_q);
            ++nq;
          }
        }
        for (int t = 0; t < w.n && !*abort_flag; ++t, ++T) {
          const int s = int(T % ST);
          if (T >= ST && !mbar_wait_sleep(empty0 + 8u * s, int((T / ST) - 1) & 1, abort_flag)) {
            *abort_flag = 1; report_fault(p.err, 5, code); break;
          }
          const int32_t j = __ldg(p.col_idx + w.start + t);
          mbar_arrive_expect_tx(full0 + 8u * s, C::KV_BYTES);
          for (int c = 0; c < D / 64; ++c)
            load_rows(ring + s * C::KV_BYTES + c * BN * 128, tmap, c, w.plane, int64_t(j) * BN, full0 + 8u * s);
        }
      }
      __syncwarp();
    }
    if (lane == 0 && *abort_flag) {
      for (uint32_t u = (T > uint32_t(ST) ? T - ST : 0); u < T; ++u)
        mbar_wait(full0 + 8u * int(u % ST), int(u / ST) & 1, never);
      if (with_q && nq > 0) mbar_wait(bar_q, (nq - 1) & 1, never);
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer: Q, K
    if (lane == 0) { tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); }
    produce(&tm_k, sK, C::KST, bar_k_full(0), bar_k_empty(0), 1, true);
  } else if (warp == kVWarp) {
    // ------------------------------------------------------------ TMA producer: V
    if constexpr (!LSE_ONLY) {
      if (lane == 0) tma_prefetch_desc(&tm_v);
      produce(&tm_v, sV, C::VST, bar_v_full(0), bar_v_empty(0), 6, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer: S = Q K^T
    // S(T+2) is issued as soon as the softmax has read S(T) (same S buffer).  O += P V is
    // issued by its own warp, so neither issue stream waits behind the other's barriers;
    // the two write disjoint TMEM columns and read disjoint shared memory.  Descriptors are
    // built once; an MMA only adds a byte offset / 16 to the start-address field (shared
    // addresses stay below 2^18 bytes, so the 14-bit field never carries).
    const uint64_t q_desc = smem_desc_sw128(sQ, 16, 1024);
    const uint64_t k_desc = smem_desc_sw128(sK, 16, 1024);
    bool ok = true, any_mma = false;
    uint32_t T = 0;
    int nq = 0;
    for (int it = it_begin; ok && it < it_end; ++it) {
      const Item w = item_at(it);
      if (w.n == 0) continue;
      if (lane == 0) {
        ok = mbar_wait_sleep(bar_q, nq & 1, abort_flag);
        for (int t = 0; ok && t < w.n; ++t, ++T) {
          const int s = int(T % C::KST), b = int(T % C::NSB);
          if (!mbar_wait_sleep(bar_k_full(s), int(T / C::KST) & 1, abort_flag)) { ok = false; break; }
          // S_b is free again: read by the softmax (LSE only), or read and overwritten with P
          // and that P read by O += P V (the P V of position T - NSB)
          if (T >= uint32_t(C::NSB) &&
              !mbar_wait_sleep(LSE_ONLY ? bar_s_free(b) : bar_o_done(b), int((T / C::NSB) - 1) & 1, abort_flag)) {
            ok = false; break;
          }
          tc_fence_after();
          const uint64_t ks = k_desc + uint64_t((s * C::KV_BYTES) >> 4);
          const uint32_t s_tm = tmem + C::TM_S + 128 * b;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_f16_ss(s_tm, q_desc + uint64_t(((kk / 4) * BM * 128 + (kk % 4) * 32) >> 4),
                        ks + uint64_t(((kk / 4) * BN * 128 + (kk % 4) * 32) >> 4), C::IDESC_QK,
                        kk > 0 ? 1u : 0u);
          umma_commit(bar_s_full(b));
          umma_commit(bar_k_empty(s));
          any_mma = true;
        }
        // Q may be replaced once this item's Q K^T MMAs have completed.
        if (ok) umma_commit(bar_q_empty);
        ++nq;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (lane == 0) {
      if (!ok) { *abort_flag = 1; report_fault(p.err, 5, 2); }
      if (any_mma) {
        // Drain: every MMA issued by this thread completes before TMEM is released.
        umma_commit(bar_final);
        mbar_wait(bar_final, 0, never);
      }
    }
  } else if (warp == kPVWarp) {
    if constexpr (!LSE_ONLY) {
      // ------------------------------------------------------------ MMA issuer: O += P V
      // O += P(T) V_T as soon as P(T) is in TMEM and V_T has landed; P is the TMEM A operand.
      // An item's first P V overwrites O, so it waits until the softmax warps have read the
      // previous item's O in their epilogue.
      const uint64_t v_desc = smem_desc_sw128(sV, BN * 128, 1024);
      bool ok = true, any_mma = false;
      uint32_t T = 0;
      int nq = 0;
      for (int it = it_begin; ok && it < it_end; ++it) {
        const Item w = item_at(it);
        if (w.n == 0) continue;
        if (lane == 0) {
          if (nq > 0) ok = mbar_wait_sleep(bar_o_free, (nq - 1) & 1, abort_flag);
          for (int t = 0; ok && t < w.n; ++t, ++T) {
            const int s = int(T % C::VST), b = int(T % C::NSB);
            if (!mbar_wait_sleep(bar_p_full(b), int(T / C::NSB) & 1, abort_flag)) { ok = false; break; }
            if (!mbar_wait_sleep(bar_v_full(s), int(T / C::VST) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint64_t vs = v_desc + uint64_t((s * C::KV_BYTES) >> 4);
            const uint32_t p_tm = tmem + C::TM_S + 128 * b;
  #pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              umma_f16_ts(tmem + C::TM_O, p_tm + kk * 8, vs + uint64_t((kk * 16 * 128) >> 4), C::IDESC_PV,
                          (t > 0 || kk > 0) ? 1u : 0u);
            umma_commit(bar_v_empty(s));
            umma_commit(bar_o_done(b));
            any_mma = true;
          }
          ++nq;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
      if (lane == 0) {
        if (!ok) { *abort_flag = 1; report_fault(p.err, 5, 7); }
        if (any_mma) {
          umma_commit(bar_final_pv);
          mbar_wait(bar_final_pv, 0, never);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Thread = (query row, column half).  The warp may access TMEM lane quarter w & 3 and
    // takes 16 of its 32 lanes; with the .16x32bx2 shapes lane t (t < 16) moves columns
    // [0, half) of row base + t and lane t + 16 columns [half, 2 half) of the same row.
    constexpr int HALF = BN / 2, DH = D / 2;
    const int quarter = warp & 3;                 // TMEM lane quarter this warp may access
    const int sel = (warp - kSoftmaxWarp0) >> 2;  // which 16 lanes of the quarter
    const int hf = lane >> 4;                     // column half
    const int row = quarter * 32 + sel * 16 + (lane & 15);   // row of the 128-row tile
    const uint32_t lane_off = uint32_t(quarter * 32 + sel * 16) << 16;
    const float c = p.scale_log2;                 // scores -> log2 units
    bool ok = true;
    uint32_t T = 0;
    int nq = 0;
    for (int it = it_begin; ok && it < it_end; ++it) {
      const Item w = item_at(it);
      if (w.skip) continue;
      const int n = w.n;
      if (w.bad && warp == kSoftmaxWarp0 && lane == 0)
        report_fault(p.err, 1, (p.mask_heads == 1 ? 0 : w.plane % p.H) * p.nb + w.i);
      float m_ref = -INFINITY;                    // running max in log2 units (lazy)
      float l = 0.f;                              // this half's share of the row sum
      // Key blocks j >= n_valid / Bs hold padding keys: the block holding the sequence end and
      // any block of padding only (possible when n_pad - n_valid >= Bs).  CSR rows ascend, so
      // they are the row's last entries: entries [0, t_tail) take the step without padding
      // code, entries [t_tail, n) the masked step.  (Every lane reads the same entries.)
      const int64_t j_part = p.n_valid / BN;
      int t_tail = n;
      while (t_tail > 0 && int64_t(__ldg(p.col_idx + w.start + t_tail - 1)) >= j_part) --t_tail;

      // One key block t (pipeline position T); false when a wait gives up.
      auto step = [&](int t, auto masked_tag) -> bool {
        constexpr bool MASKED = decltype(masked_tag)::value;
        const int b = int(T % C::NSB);
        if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full(b), int(T / C::NSB) & 1, abort_flag))) return false;
        tc_fence_after();
        uint32_t sr[HALF];
#pragma unroll
        for (int q = 0; q < HALF / 32; ++q)
          tmem_ld_16x2_32<HALF>(tmem + lane_off + C::TM_S + 128 * b + q * 32,
                                *reinterpret_cast<uint32_t(*)[32]>(sr + q * 32));
        tmem_wait_ld();
        if constexpr (LSE_ONLY) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_s_free(b));
        }
        // Masked step: the real keys of this half.  Scores of padding keys become a sentinel
        // whose scaled value is -inf (its exponential is 0, or 2^-125 on the FMA-pipe path:
        // nothing next to a real key's); a block of padding only stores P = 0 and adds
        // nothing.  The choice is the whole warp's: the key block is the same for every lane.
        bool any_key = true;
        if constexpr (MASKED) {
          const int64_t valid_blk = p.n_valid - int64_t(__ldg(p.col_idx + w.start + t)) * BN;
          any_key = valid_blk > 0;
          if (any_key) {
            const int64_t valid = valid_blk - hf * HALF;
            const uint32_t sentinel = __float_as_uint(NEG ? INFINITY : -INFINITY);
#pragma unroll
            for (int e = 0; e < HALF; ++e)
              if (e >= valid) sr[e] = sentinel;
          }
        }
        float mx = -INFINITY;
        if (any_key) {
          // max of s*c is c*max(s) for c >= 0 and c*min(s) otherwise (3-input max, 4 chains)
          float m4[4];
          if constexpr (!NEG) {
#pragma unroll
            for (int e = 0; e < 4; ++e) m4[e] = -INFINITY;
#pragma unroll
            for (int e = 0; e < HALF / 2; ++e)
              m4[e & 3] = fmax3(m4[e & 3], __uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]));
            mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * c;
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) m4[e] = INFINITY;
#pragma unroll
            for (int e = 0; e < HALF / 2; ++e)
              m4[e & 3] = fmin3(m4[e & 3], __uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]));
            mx = fminf(fminf(m4[0], m4[1]), fminf(m4[2], m4[3])) * c;
          }
        }
        // Row max over both halves (lanes t and t ^ 16 hold one row).
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_old = m_ref;
        if (mx > m_ref + kRescaleThreshold || m_ref == -INFINITY) m_ref = fmaxf(mx, m_ref);
        const float alpha = (m_old == m_ref) ? 1.f : ex2_approx(m_old - m_ref);
        const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        // P(t) goes over S(t)'s first columns, which every lane of the warp has loaded (the
        // row-max shuffle above follows each lane's load wait).
        __syncwarp();
        const uint32_t p_tm = tmem + lane_off + C::TM_S + 128 * b;
        float r4[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[HALF / 2];
        if (any_key) {
          // Pairs of elements with packed fp32 math; the pairs kPolyPair picks take their
          // exponentials on the FMA pipe, the rest on the MUFU.  With 64-key halves the first
          // 16 pairs go to TMEM while the rest are computed.
          const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m_use, -m_use);
          uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
          for (int e = 0; e < HALF / 2; ++e) {
            const uint64_t x2 = f2_fma(f2_pack_bits(sr[2 * e], sr[2 * e + 1]), c2, nm2);
            uint64_t p2;
            if (kPolyPair<LSE_ONLY>(e)) {
              p2 = exp2_poly_f2(x2);
            } else {
              float x0, x1;
              f2_unpack(x2, x0, x1);
              p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
            }
            acc[e & 1] = f2_add(acc[e & 1], p2);
            if constexpr (!LSE_ONLY) {
              float p0, p1;
              f2_unpack(p2, p0, p1);
              pk[e] = pack_bf16x2(p0, p1);
              if constexpr (HALF == 64) {
                if (e == 15) tmem_st_16x2_16<HALF / 2>(p_tm, *reinterpret_cast<const uint32_t(*)[16]>(pk));
              }
            }
          }
          if constexpr (!LSE_ONLY) {
            if constexpr (HALF == 64) {
              tmem_st_16x2_16<HALF / 2>(p_tm + 16, *reinterpret_cast<const uint32_t(*)[16]>(pk + 16));
            } else {
              tmem_st_16x2_16<HALF / 2>(p_tm, *reinterpret_cast<const uint32_t(*)[16]>(pk));
            }
          }
          float a0, a1, b0, b1;
          f2_unpack(acc[0], a0, a1);
          f2_unpack(acc[1], b0, b1);
          r4[0] = a0; r4[1] = a1; r4[2] = b0; r4[3] = b1;
        } else if constexpr (!LSE_ONLY) {
#pragma unroll
          for (int e = 0; e < HALF / 2; ++e) pk[e] = 0u;
          if constexpr (HALF == 64) {
            tmem_st_16x2_32<HALF / 2>(p_tm, *reinterpret_cast<const uint32_t(*)[32]>(pk));
          } else {
            tmem_st_16x2_16<HALF / 2>(p_tm, *reinterpret_cast<const uint32_t(*)[16]>(pk));
          }
        }
        l = l * alpha + ((r4[0] + r4[1]) + (r4[2] + r4[3]));

        // O was last written by O += P(t-1) V: rescale it (rarely) once that has completed,
        // before P(t) is released to the P V issuer.
        if (!LSE_ONLY && t >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
          if (!__all_sync(0xffffffffu, mbar_wait(bar_o_done(int((T - 1) % C::NSB)), int((T - 1) / C::NSB) & 1, abort_flag))) {
            return false;
          }
          tc_fence_after();
          rescale_o<DH>(tmem + lane_off + C::TM_O, alpha);
        }
        if constexpr (!LSE_ONLY) {
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_p_full(b));
        }
        return true;
      };

      // Speculative step for a full key block after the item's first: the exponentials are
      // taken against the current reference max while the block max is computed alongside,
      // so no max -> exponentials dependency is on the path.  When some row's block max
      // exceeds its reference by more than the rescale threshold (rare once the first block
      // has set it), the block is given up before S or P is released and the max-first step
      // redoes it; otherwise the results are the max-first step's, bit for bit (same reference,
      // same arithmetic).  Returns 0 when a wait gives up, 1 when done, 2 for a redo.
      auto step_spec = [&](int t) -> int {
        (void)t;
        const int b = int(T % C::NSB);
        if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full(b), int(T / C::NSB) & 1, abort_flag))) return 0;
        tc_fence_after();
        uint32_t sr[HALF];
#pragma unroll
        for (int q = 0; q < HALF / 32; ++q)
          tmem_ld_16x2_32<HALF>(tmem + lane_off + C::TM_S + 128 * b + q * 32,
                                *reinterpret_cast<uint32_t(*)[32]>(sr + q * 32));
        tmem_wait_ld();
        const uint32_t p_tm = tmem + lane_off + C::TM_S + 128 * b;
        const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m_ref, -m_ref);
        uint64_t acc[2] = {0ull, 0ull};
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        uint32_t pk[HALF / 2];
#pragma unroll
        for (int e = 0; e < HALF / 2; ++e) {
          m4[e & 3] = fmax3(m4[e & 3], __uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]));
          const uint64_t x2 = f2_fma(f2_pack_bits(sr[2 * e], sr[2 * e + 1]), c2, nm2);
          uint64_t p2;
          if (kPolyPair<LSE_ONLY>(e)) {
            p2 = exp2_poly_f2(x2);
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
          }
          acc[e & 1] = f2_add(acc[e & 1], p2);
          if constexpr (!LSE_ONLY) {
            float p0, p1;
            f2_unpack(p2, p0, p1);
            pk[e] = pack_bf16x2(p0, p1);
          }
        }
        float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * c;
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        // A redo reloads S, so P (which goes over S) is stored only once the block commits.
        if (__any_sync(0xffffffffu, mx > m_ref + kRescaleThreshold || m_ref == -INFINITY)) return 2;
        if constexpr (!LSE_ONLY) {
          if constexpr (HALF == 64) {
            tmem_st_16x2_32<HALF / 2>(p_tm, *reinterpret_cast<const uint32_t(*)[32]>(pk));
          } else {
            tmem_st_16x2_16<HALF / 2>(p_tm, *reinterpret_cast<const uint32_t(*)[16]>(pk));
          }
          tmem_wait_st();
        }
        float a0, a1, b0, b1;
        f2_unpack(acc[0], a0, a1);
        f2_unpack(acc[1], b0, b1);
        l = l + ((a0 + a1) + (b0 + b1));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (LSE_ONLY) mbar_arrive(bar_s_free(b));
          else mbar_arrive(bar_p_full(b));
        }
        return 1;
      };
      for (int t = 0; ok && t < t_tail; ++t, ++T) {
        int r = 2;
        if constexpr (!NEG) {
          if (t > 0) r = step_spec(t);
        }
        if (r == 0) ok = false;
        else if (r == 2) ok = step(t, std::false_type{});
      }
      for (int t = t_tail; ok && t < n; ++t, ++T) ok = step(t, std::true_type{});
      if (!ok) break;

      // ---------------------------------------------------------- epilogue of this item
      const int64_t plane = w.plane;
      const int i = w.i;
      const int64_t grow = int64_t(i) * BN + row;           // row within the plane
      const bool store = row < BN && grow < p.n_pad;
      const float l_row = l + __shfl_xor_sync(0xffffffffu, l, 16);
      const bool have = n > 0 && l_row > 0.f;
      if constexpr (!LSE_ONLY) {
        // O row destination: tile order, or (fused inverse reorder) the row's raster position;
        // padding rows have no raster position and are not written then.
        __nv_bfloat16* orow;
        bool store_o = store;
        if (p.o_raster != nullptr) {
          store_o = store && grow < p.n_valid;
          const uint32_t raster = store_o ? tile_order_to_raster(uint32_t(grow), p.grid) : 0u;
          orow = p.o_raster + (plane * p.n_valid + int64_t(raster)) * D + hf * DH;
        } else {
          orow = p.o + (plane * p.n_pad + grow) * D + hf * DH;
        }
        const float inv_l = have ? 1.f / l_row : 0.f;
        if (n > 0) {
          const uint32_t T_last = T - 1;
          if (!__all_sync(0xffffffffu, mbar_wait(bar_o_done(int(T_last % C::NSB)), int(T_last / C::NSB) & 1, abort_flag))) {
            ok = false; break;
          }
          tc_fence_after();
        }
  #pragma unroll 1
        for (int q = 0; q < DH / 32; ++q) {
          uint32_t ov[32];
          if (n > 0) {
            tmem_ld_16x2_32<DH>(tmem + lane_off + C::TM_O + q * 32, ov);
            tmem_wait_ld();
            if (q == DH / 32 - 1) {
              // All of O is in registers: the next item's first P V may overwrite it.
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(bar_o_free);
            }
          }
          if (store_o) {
            if (p.o_align32) {
  #pragma unroll
              for (int e8 = 0; e8 < 2; ++e8) {
                uint32_t w8[8];
  #pragma unroll
                for (int e = 0; e < 8; ++e)
                  w8[e] = have ? pack_bf16x2(__uint_as_float(ov[16 * e8 + 2 * e]) * inv_l,
                                             __uint_as_float(ov[16 * e8 + 2 * e + 1]) * inv_l) : 0u;
                st_global_v8(orow + q * 32 + e8 * 16, w8);
              }
            } else {
  #pragma unroll
              for (int e4 = 0; e4 < 4; ++e4) {
                uint32_t w4[4];
  #pragma unroll
                for (int e = 0; e < 4; ++e)
                  w4[e] = have ? pack_bf16x2(__uint_as_float(ov[8 * e4 + 2 * e]) * inv_l,
                                             __uint_as_float(ov[8 * e4 + 2 * e + 1]) * inv_l) : 0u;
                reinterpret_cast<uint4*>(orow + q * 32)[e4] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
              }
            }
          }
        }
      }
      if (n > 0) ++nq;
      if (store && hf == 0)
        p.lse[plane * p.n_pad + grow] = have ? (m_ref + __log2f(l_row)) * 0.69314718055994530942f : -INFINITY;
    }
    if (!ok) { *abort_flag = 1; if (lane == 0) report_fault(p.err, 5, 3); }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int BN, int KPC, bool LSE_ONLY, bool NEG>
cudaError_t launch_cfg(const AttnArgs& a, cudaStream_t stream, const char** why) {
  using C = Cfg<D, BN, LSE_ONLY>;
  const int64_t rows = int64_t(a.B) * a.H * a.n_pad;
  CUtensorMap tq, tk, tv;
  bool maps_ok;
  if (a.gather_windows == 0) {
    maps_ok = make_rows_map(&tq, a.q, rows, D, BM) && make_rows_map(&tk, a.k, rows, D, BN) &&
              make_rows_map(&tv, LSE_ONLY ? a.k : a.v, rows, D, BN);
  } else {
    const int64_t planes = int64_t(a.B) * a.H;
    maps_ok = make_window_gather_map(&tq, a.q, planes, a.gather_windows, a.gather_window, D, BM) &&
              make_window_gather_map(&tk, a.k, planes, a.gather_windows, a.gather_window, D, BN) &&
              make_window_gather_map(&tv, LSE_ONLY ? a.k : a.v, planes, a.gather_windows, a.gather_window, D, BN);
  }
  if (!maps_ok) {
    *why = "cuTensorMapEncodeTiled failed or is unavailable";
    return cudaErrorInvalidValue;
  }
  static DeviceFlags attr_set = {};
  cudaError_t e = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(bsa_fwd_kernel<D, BN, KPC, LSE_ONLY, NEG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::SMEM_BYTES);
  });
  if (e != cudaSuccess) { *why = "cudaFuncSetAttribute(max dynamic smem) failed"; return e; }
  AttnParams p;
  p.H = a.H;
  p.nb = int(a.n_pad / a.block_size);
  p.mask_heads = a.mask_heads;
  p.n_pad = a.n_pad;
  p.n_valid = a.n_valid;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.row_ptr = a.row_ptr;
  p.col_idx = a.col_idx;
  p.col_len = a.col_len;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.o_raster = static_cast<__nv_bfloat16*>(a.o_raster);
  p.grid = Grid3{uint32_t(a.T), uint32_t(a.Hg), uint32_t(a.Wg), uint32_t(a.tt), uint32_t(a.th),
                 uint32_t(a.tw)};
  p.gather_windows = a.gather_windows;
  p.o_align32 = ((reinterpret_cast<uintptr_t>(a.o_raster != nullptr ? a.o_raster : a.o) & 31) == 0) ? 1 : 0;
  p.lse = a.lse;
  p.query_src = a.query_src;
  p.src_heads = a.src_heads;
  p.err = a.err;
  const int64_t items = rows / a.block_size;
  if (items == 0) return cudaSuccess;
  p.items = items;
  const int64_t grid = (items + KPC - 1) / KPC;
  bsa_fwd_kernel<D, BN, KPC, LSE_ONLY, NEG><<<dim3(unsigned(grid)), kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

// Query blocks per CTA.  A CTA walks a run of consecutive query blocks: its prologue
// (barriers, TMEM allocation, the first Q and K tiles) is paid once per run and the next
// block's loads and first Q K^T overlap the current epilogue, while the hardware still hands
// out runs in order as SMs free up.  That pays off for short CSR rows (a few key blocks per
// query block) and costs tail balance and L2 locality for long ones.  With col_len taken as
// the entry count: runs of 8 for rows averaging at most 3 key blocks, 4 for at most 8,
// otherwise 1 (a capacity larger than the entry count therefore selects 1).
template <int D, int BN, bool LSE_ONLY>
cudaError_t launch_dispatch(const AttnArgs& a, cudaStream_t stream, const char** why) {
  // A negative softmax scale (rare) takes its own instantiation, one query block per CTA.
  if (a.scale < 0.f) return launch_cfg<D, BN, 1, LSE_ONLY, true>(a, stream, why);
  const int64_t rows = int64_t(a.mask_heads) * (a.n_pad / a.block_size);
  if (rows > 0 && a.col_len <= 3 * rows) return launch_cfg<D, BN, 8, LSE_ONLY, false>(a, stream, why);
  if (rows > 0 && a.col_len <= 8 * rows) return launch_cfg<D, BN, 4, LSE_ONLY, false>(a, stream, why);
  return launch_cfg<D, BN, 1, LSE_ONLY, false>(a, stream, why);
}

cudaError_t launch_attn(const AttnArgs& a, cudaStream_t stream, const char** why) {
  if (a.lse_only) {
    // LSE only (lva_block_sparse_lse): no V, no P V product, no O
    if (a.d == 128 && a.block_size == 128) return launch_dispatch<128, 128, true>(a, stream, why);
    if (a.d == 128 && a.block_size == 64) return launch_dispatch<128, 64, true>(a, stream, why);
    if (a.d == 64 && a.block_size == 128) return launch_dispatch<64, 128, true>(a, stream, why);
    if (a.d == 64 && a.block_size == 64) return launch_dispatch<64, 64, true>(a, stream, why);
  } else {
    if (a.d == 128 && a.block_size == 128) return launch_dispatch<128, 128, false>(a, stream, why);
    if (a.d == 128 && a.block_size == 64) return launch_dispatch<128, 64, false>(a, stream, why);
    if (a.d == 64 && a.block_size == 128) return launch_dispatch<64, 128, false>(a, stream, why);
    if (a.d == 64 && a.block_size == 64) return launch_dispatch<64, 64, false>(a, stream, why);
  }
  *why = "unsupported (d, block_size)";
  return cudaErrorInvalidValue;
}

}  // namespace lva

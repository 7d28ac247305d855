/*
 * lva.h -- block-sparse softmax attention for video diffusion transformers on B200 (sm_100a).
 *
 * C ABI.  Every pointer argument named as "device" is a device address of the current CUDA
 * device; every call is asynchronous on the given stream and returns after argument checks
 * and kernel launch.  The library allocates no memory: the caller owns every buffer.
 *
 * Errors: a call returns LVA_OK or a status code.  Argument errors are found on the host
 * before anything is launched (nothing is written in that case).  A failed launch returns
 * LVA_ERR_CUDA.  Faults found by the kernels themselves (a CSR entry out of range, a wait
 * that ran past its time limit) are recorded in a per-device error word that
 * lva_device_error() reads; the kernels then skip the bad work instead of touching memory
 * outside the buffers.  lva_last_error_message() gives a one-line explanation of the
 * last failure on the calling thread.
 *
 * Layouts:
 *   tokens   -- a plane (one batch element and head) is n rows of row_elems elements;
 *               planes are contiguous: element (p, r, e) sits at ((p*n + r)*row_elems + e).
 *   Q, K, V, O -- bf16 [B, H, n_pad, d], row-major, rows in tile order (see
 *               lva_reorder_tokens), rows n_valid..n_pad-1 are padding.
 *   LSE      -- fp32 [B, H, n_pad].
 *   CSR      -- row r = h_m*nb + i lists the key blocks j that query block i attends under
 *               mask head h_m: col_idx[row_ptr[r] .. row_ptr[r+1]-1], ascending, unique.
 */
#ifndef LVA_H
#define LVA_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LVA_VERSION 1

typedef enum {
  LVA_OK = 0,
  LVA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, inconsistent sizes, bad CSR */
  LVA_ERR_UNSUPPORTED = 2,   /* a size or mode the library has no kernel for */
  LVA_ERR_CAPACITY = 3,      /* an output buffer is too small */
  LVA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  LVA_ERR_TIMEOUT = 5        /* a kernel wait ran past its limit (device error word) */
} lva_status;

/* Human-readable name of a status code (static string). */
const char* lva_status_string(lva_status status);

/* One-line description of the last failure on the calling thread ("" if none). */
const char* lva_last_error_message(void);

/* LVA_VERSION of the loaded library. */
int lva_version(void);

/*
 * lva_reorder_tokens -- spatiotemporal-tile token order and its inverse.
 *
 * Defines the token order in which blocks of the attention matrix are spatiotemporal
 * neighbourhoods, the granularity at which the LVSA page ("LVSA: Training-Free Sparse
 * Attention for Long Video Diffusion", technical summary section 2, "Meccanismo Core")
 * restricts a query frame's attended set, and at which the CalibAtt page ("Accelerating
 * Text-to-Video Generation with Calibrated Sparse Attention", section 2, step A.1) cuts
 * the matrix into 128x128 blocks.  The order: tiles of tile_t x tile_h x tile_w latent
 * tokens, enumerated in raster order of tile coordinates; tokens in raster order inside a
 * tile; edge tiles are partial (no per-tile padding).
 *
 * With N = T*H*W and perm[k] the raster index t*H*W + h*W + w of the k-th token in tile
 * order:
 *   inverse == 0:  src [planes, N, row] (raster) -> dst [planes, n_pad, row] (tile order):
 *                  dst[p][k] = src[p][perm[k]] for k < N; rows N..n_pad-1 are zeroed.
 *   inverse != 0:  src [planes, n_pad, row] (tile order) -> dst [planes, N, row] (raster):
 *                  dst[p][perm[k]] = src[p][k] for k < N; src rows >= N are ignored.
 * Rows are copied bit for bit.  row = row_elems elements of elem_bytes (2 or 4) bytes.
 *
 * src, dst: device, must not overlap, aligned to elem_bytes.  n_pad >= N.
 * planes * n_pad * row_elems * elem_bytes must fit in int64.
 * Errors: LVA_ERR_INVALID_ARG for null pointers, non-positive sizes, n_pad < N, bad
 * elem_bytes or misalignment.  LVA_ERR_UNSUPPORTED when N or n_pad reaches 2^31, a row
 * exceeds 1 MiB, or n_pad * row_elems exceeds (2^31 - 1) * 256, the most one launch
 * covers.  planes == 0 is a no-op once the sizes have been checked.
 */
lva_status lva_reorder_tokens(const void* src, void* dst, int64_t planes,
                              int T, int H, int W, int tile_t, int tile_h, int tile_w,
                              int64_t n_pad, int64_t row_elems, int elem_bytes, int inverse,
                              cudaStream_t stream);

/* Block-mask kinds for lva_build_block_mask. */
typedef enum {
  LVA_MASK_WINDOW_ANCHOR = 0,  /* local window + rotating global anchors (LVSA)      */
  LVA_MASK_STATIC = 1,         /* a given dense per-head block mask (CalibAtt-style) */
  LVA_MASK_ALL = 2,            /* every block: dense attention                       */
  LVA_MASK_TWO_STAGE = 3,      /* local window groups + one strided block (SQuad-style) */
  LVA_MASK_LVSA_FRAMES = 4     /* expanded frame windows + rotating global frames (LVSA) */
} lva_mask_kind;

typedef struct {
  int kind;                    /* lva_mask_kind */
  int mask_heads;              /* H_m: rows of masks built; 1 unless kind is STATIC */
  int block_size;              /* Bs: 64 or 128 tokens */
  int64_t n_pad;               /* padded sequence length, a multiple of block_size */
  int64_t n_valid;             /* real tokens, 1 <= n_valid <= n_pad */
  int64_t window_unit_tokens;  /* WINDOW_ANCHOR: U, tokens per window unit (H*W = frames) */
  int window_radius;           /* WINDOW_ANCHOR: r >= 0, in units */
  int num_anchors;             /* WINDOW_ANCHOR: G >= 0 anchor key blocks */
  int step;                    /* WINDOW_ANCHOR: denoising step s >= 0 */
  int group_blocks;            /* TWO_STAGE: g >= 1 blocks per local window group */
  int budget_frames;           /* LVSA_FRAMES: C >= 1 attended frames per query frame */
} lva_mask_params;

/* Upper bound on the CSR entries of a mask: mask_heads * nb * nb (0 on bad params). */
int64_t lva_block_mask_max_nnz(const lva_mask_params* params);

/*
 * lva_build_block_mask -- per-query-block CSR lists of the key blocks to compute.
 *
 * The CSR is the skip list of the CalibAtt page ("Accelerating Text-to-Video Generation
 * with Calibrated Sparse Attention", section 2 B, "Fase di Inferenza": precomputed lists of
 * blocks per (timestep, layer, head), deterministic, no decision at inference time), built
 * on the GPU from one of these masks, with nb = n_pad / block_size:
 *
 *   WINDOW_ANCHOR (LVSA page, technical summary section 2, "Meccanismo Core":
 *     A(t) = G union W(t); the global set G_s moves by s mod T_per at step s).
 *     Block i covers window units lo(i) = floor(i*Bs/U) .. hi(i) = floor((min((i+1)*Bs,
 *     n_valid) - 1)/U); a block of padding only takes the unit of the last real token.
 *     Anchors G_s = { (floor(a*nb/G) + s) mod nb : a < G }.
 *     M[i][j] = (lo(j) <= hi(i) + r  and  hi(j) >= lo(i) - r)  or  j in G_s.
 *   STATIC: M[h][i][j] = dense_mask[(h*nb + i)*nb + j] != 0, used as given.
 *   ALL:    M[i][j] = 1.
 *   TWO_STAGE (SQuad page, "SQuad: Sub-Quadratic Attention Distillation for Efficient
 *     Video Generation", technical summary section 1: local pass in windows of w tokens,
 *     global pass across windows at the same relative position):
 *     M[i][j] = (floor(j/g) == floor(i/g))  or  j == (i + g) mod nb.
 *   LVSA_FRAMES (LVSA page, technical summary section 2, "Ancore Globali Rotanti" and
 *     "Finestre Adattive Espanse": global frames rotate with the step; the local window is
 *     extended where it overlaps global frames so that a query frame attends C frames).
 *     Frames f = 0..T-1 of U = window_unit_tokens tokens, T = ceil(n_valid / U); global
 *     frames G_s = { (floor(a*T/G) + s) mod T : a < G }.  W(t) starts as {t} and grows one
 *     frame at a time, right then left alternately (the other side when one end is reached),
 *     until |G_s union W(t)| = min(C, T); A(t) = G_s union W(t).  Query block i attends key
 *     block j when a frame of j lies in A(t) for a frame t of i (frames of real tokens; a
 *     padding-only block takes the last frame).
 *
 * Outputs (device): row_ptr [mask_heads*nb + 1] (row_ptr[0] = 0), col_idx [col_capacity],
 * *nnz_out = row_ptr[mask_heads*nb].  Columns of a row are ascending and unique.
 * dense_mask (device) is read only for STATIC ([mask_heads, nb, nb] uint8) and may be NULL
 * otherwise.
 * Errors: LVA_ERR_INVALID_ARG for bad parameters or pointers; LVA_ERR_UNSUPPORTED for a
 * block_size other than 64 or 128, or mask_heads*nb*nb >= 2^31 (the CSR's int32 entries);
 * LVA_ERR_CAPACITY when col_capacity < lva_block_mask_max_nnz(params).  Nothing is
 * launched in any of these cases.
 */
lva_status lva_build_block_mask(const lva_mask_params* params, const uint8_t* dense_mask,
                                int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                int32_t* nnz_out, cudaStream_t stream);

/*
 * lva_block_mask_workspace_bytes -- device workspace of lva_build_block_mask_ws.
 *
 * Bytes of the caller-owned workspace that lva_build_block_mask_ws needs for these
 * parameters: for STATIC, one bit per block pair (mask_heads * nb rows of
 * ceil(nb / 128) * 16 bytes), 4 bytes per row and 4 bytes per 4096 rows (each rounded up to
 * 16 bytes); 0 for the parametric kinds.
 * Returns -1 for invalid parameters.
 */
int64_t lva_block_mask_workspace_bytes(const lva_mask_params* params);

/*
 * lva_build_block_mask_ws -- lva_build_block_mask with a caller-owned device workspace.
 *
 * The same CSR, bit for bit, as lva_build_block_mask.  For STATIC masks the dense input is
 * read once: a first pass writes every row as bits (into `workspace`) and its count, the
 * counts are scanned (by several CTAs when there are more than 4096 rows), and a last pass
 * expands the bits into the column lists.  lva_build_block_mask reads the dense mask twice
 * instead (a count pass and a fill pass) and needs no workspace.  The parametric kinds need
 * none here either (workspace may then be NULL).
 *
 * workspace: device, 16-byte aligned, at least lva_block_mask_workspace_bytes(params)
 * bytes (its contents are overwritten; it may be reused once the call has completed on
 * `stream`).  Other arguments and errors as for lva_build_block_mask; in addition
 * LVA_ERR_INVALID_ARG for a null or misaligned workspace and LVA_ERR_CAPACITY when
 * workspace_bytes is too small.
 */
lva_status lva_build_block_mask_ws(const lva_mask_params* params, const uint8_t* dense_mask,
                                   int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                   int32_t* nnz_out, void* workspace, int64_t workspace_bytes,
                                   cudaStream_t stream);

/*
 * lva_build_block_mask_noalloc -- lva_build_block_mask_ws without a caller workspace.
 *
 * An addition of this library; the pages have no counterpart.  For callers that cannot
 * allocate device memory at all: code that runs inside a host framework which owns every
 * device allocation and hands its plugins only their input and output buffers, or a
 * real-time path with a fixed memory budget where no allocation may happen after start-up.
 * This call builds the same CSR, bit for bit, as lva_build_block_mask_ws, with that call's
 * workspace taken from a 16 MiB array that the library itself places in device memory: it
 * calls no cudaMalloc, cudaFree or other allocating routine.  The caller still passes the
 * mask and the CSR outputs (arguments and errors as for lva_build_block_mask).
 *
 * Limit: lva_block_mask_workspace_bytes(params) must be at most 16 MiB (16777216 bytes;
 * for STATIC masks about 128 Mi block pairs, e.g. 4 heads of 4096 x 4096 blocks), else
 * LVA_ERR_CAPACITY is returned and nothing is launched.  The parametric kinds need no
 * scratch.  Every device that loads the library holds the 16 MiB until the process exits.
 * The first call on a device looks up the array's device address (a runtime call, done once
 * per device with that device current); make that first call before any stream capture.
 * All calls share the one array, so calls whose work overlaps on the GPU (other streams,
 * other host threads) race and must be ordered by the caller; the array keeps the last
 * call's contents, and a call reads only what it has written itself.
 */
lva_status lva_build_block_mask_noalloc(const lva_mask_params* params, const uint8_t* dense_mask,
                                        int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                        int32_t* nnz_out, cudaStream_t stream);

/*
 * lva_block_sparse_attn -- softmax attention computed only on listed block pairs.
 *
 * The block-sparse attention of the LVSA page (technical summary section 2: attention
 * restricted to A(t) through a block-sparse mechanism) and of the CalibAtt page (section
 * 2 B: non-repetitive heads attend only the selected blocks of the skip list).  For batch
 * b, head h and query row r in block i = r / Bs, with h_m = (mask_heads == 1 ? 0 : h):
 *   J   = { c : c < n_valid and c / Bs is listed in CSR row h_m*nb + i }
 *   s_c = scale * <q_r, k_c>;  m = max_c s_c;  l = sum_c exp(s_c - m)
 *   O_r = sum_c exp(s_c - m) v_c / l   (bf16, round to nearest even)
 *   LSE_r = m + ln(l)                  (fp32, natural log, scale included)
 * An empty J gives O_r = 0 and LSE_r = -inf.  Padded query rows are computed like the rest.
 * Arithmetic: bf16 tensor-core products with fp32 accumulation; probabilities are rounded
 * to bf16 before the P*V product; softmax statistics are fp32.
 *
 * q, k, v, o: device bf16 [B, H, n_pad, d], 16-byte aligned.  lse: device fp32 [B, H, n_pad].
 * row_ptr: device [mask_heads*nb + 1]; col_idx: device, col_len entries (the kernel never
 * reads past col_len).  A CSR row that reaches outside [0, col_len), lists a block outside
 * [0, nb) or does not list strictly ascending blocks is skipped (its query rows get O = 0,
 * LSE = -inf) and reported through lva_device_error as LVA_ERR_INVALID_ARG (detail = the
 * CSR row), so no key block is ever counted twice.  col_len may be the capacity of col_idx or the
 * exact entry count; the exact count lets the call see short rows, for which each CTA then
 * processes a run of consecutive query blocks (8 when rows average at most 3 key blocks, 4
 * when at most 8; results are identical either way).
 * query_src: NULL, or device int32 [src_heads, nb] (src_heads in {1, H}): query blocks with
 * query_src[h_s*nb + i] != i are not computed here (their O/LSE are left untouched for
 * lva_broadcast_blocks to fill).
 * Supported: d in {64, 128}, block_size in {64, 128}, mask_heads in {1, H},
 * B*H*n_pad < 2^31.
 */
lva_status lva_block_sparse_attn(const void* q, const void* k, const void* v, void* o, float* lse,
                                 int B, int H, int64_t n_pad, int64_t n_valid, int d,
                                 int block_size, const int32_t* row_ptr, const int32_t* col_idx,
                                 int64_t col_len, int mask_heads, float scale,
                                 const int32_t* query_src, int src_heads, cudaStream_t stream);

/*
 * lva_block_sparse_lse -- the row log-sum-exp of block-sparse attention, without O.
 *
 * The CalibAtt page ("Accelerating Text-to-Video Generation with Calibrated Sparse
 * Attention", section 2 A.1) normalises the attention scores of every query row before
 * summing them per block; with the all-ones block list this call gives that normaliser,
 * LSE_r = m + ln(l) of lva_block_sparse_attn, for lva_block_energy.  It runs the same
 * scores, maxima and sums in the same arithmetic as lva_block_sparse_attn (so the LSE is
 * the one that call returns, up to the order of floating-point additions), but never loads
 * V and computes no P V product and no O.
 *
 * q, k: device bf16 [B, H, n_pad, d], 16-byte aligned; lse: device fp32 [B, H, n_pad]
 * (written).  CSR arguments, support and errors as for lva_block_sparse_attn (no
 * repetitive-head maps).
 */
lva_status lva_block_sparse_lse(const void* q, const void* k, float* lse, int B, int H, int64_t n_pad,
                                int64_t n_valid, int d, int block_size, const int32_t* row_ptr,
                                const int32_t* col_idx, int64_t col_len, int mask_heads, float scale,
                                cudaStream_t stream);

/*
 * lva_block_sparse_attn_raster -- lva_block_sparse_attn with O written in raster order.
 *
 * The same attention as lva_block_sparse_attn on tile-order q, k, v (same definition, same
 * arithmetic, same LSE in tile order), with the inverse token reorder fused into the output:
 * the row at tile-order position r < n_valid of plane p is stored at its raster position,
 *   o_raster[p][raster(r)][:]   with raster() the tile order of lva_reorder_tokens for the
 *                               grid T x Hg x Wg and tiles tile_t x tile_h x tile_w,
 * and padded rows (r >= n_valid) are not stored.  This is the attention and the inverse
 * reorder of one layer (LVSA page, technical summary section 2; CalibAtt page, section 2 B)
 * in one launch.
 *
 * o_raster: device bf16 [B, H, n_valid, d], 16-byte aligned (written).  Requires
 * T*Hg*Wg == n_valid and extents >= 1.  Repetitive-head maps (query_src) are not accepted
 * here: their broadcast works in tile order, so use lva_block_sparse_attn for them.  Other
 * arguments, support and errors as for lva_block_sparse_attn.
 */
lva_status lva_block_sparse_attn_raster(const void* q, const void* k, const void* v, void* o_raster,
                                        float* lse, int B, int H, int64_t n_pad, int64_t n_valid,
                                        int d, int block_size, const int32_t* row_ptr,
                                        const int32_t* col_idx, int64_t col_len, int mask_heads,
                                        float scale, int T, int Hg, int Wg, int tile_t, int tile_h,
                                        int tile_w, cudaStream_t stream);

/*
 * lva_window_transposed_attn -- block-sparse attention across windows, without a transpose.
 *
 * SQuad page ("SQuad: Sub-Quadratic Attention Distillation for Efficient Video Generation"),
 * technical summary section 1: the global pass of the two-stage operator mixes the tokens at
 * the same relative position of every window.  With windows of w tokens (m = n / w windows),
 * token a*w + p is position p of window a; the window-transposed order lists position-major,
 *   row k = p*m + a of the transposed order  <->  token a*w + p of the input,
 * so each group of m consecutive transposed rows is one position across all windows.  This
 * call computes lva_block_sparse_attn on the transposed order (CSR over its blocks, same
 * definition and arithmetic) while reading q, k, v in the input order through 3D tensor
 * maps (a box gathers the rows of consecutive windows at one position), and stores O back in
 * the input order.  LSE is in the transposed order.
 *
 * q, k, v, o: device bf16 [B, H, n, d] in the input order, 16-byte aligned (o written);
 * lse: device fp32 [B, H, n].  n = m*w with m a multiple of block_size (a block never spans
 * two positions); no padding (n_valid = n).  Other arguments and errors as for
 * lva_block_sparse_attn (no repetitive-head maps).
 */
lva_status lva_window_transposed_attn(const void* q, const void* k, const void* v, void* o, float* lse,
                                      int B, int H, int64_t n, int d, int window, int block_size,
                                      const int32_t* row_ptr, const int32_t* col_idx, int64_t col_len,
                                      int mask_heads, float scale, cudaStream_t stream);

/*
 * lva_broadcast_blocks -- fill the query blocks of repetitive heads from their anchors.
 *
 * CalibAtt page ("Accelerating Text-to-Video Generation with Calibrated Sparse Attention",
 * section 2 A.3 and B): for a head whose spatial rows repeat, attention is computed only for
 * anchor rows and the result is replicated to the other rows.  At block granularity in tile
 * order: query_src[h_s*nb + i] (h_s = (src_heads == 1 ? 0 : h)) names the block whose output
 * block i takes; query_src[h_s*nb + i] == i marks a computed (anchor) block.  Run after
 * lva_block_sparse_attn with the same query_src (which skips the non-anchor blocks):
 *   O[b][h][i*Bs + r][:] = O[b][h][src*Bs + r][:],  LSE[b][h][i*Bs + r] = LSE[b][h][src*Bs + r]
 * for every block i with src = query_src[...] != i and r < Bs.
 * o: device bf16 [B, H, n_pad, d], 16-byte aligned; lse: device fp32 [B, H, n_pad].
 * A source outside [0, nb) or one that is not itself an anchor is skipped and reported
 * through lva_device_error as LVA_ERR_INVALID_ARG (detail = the offending map entry index).
 */
lva_status lva_broadcast_blocks(void* o, float* lse, int B, int H, int64_t n_pad, int d,
                                int block_size, const int32_t* query_src, int src_heads,
                                cudaStream_t stream);

/*
 * lva_block_energy -- block energies of softmax attention (static-mask calibration).
 *
 * CalibAtt page ("Accelerating Text-to-Video Generation with Calibrated Sparse Attention",
 * section 2 A.1): the attention matrix is divided into Bs x Bs blocks and, for every query
 * block, the energy toward a key block is the sum of its attention scores.  For batch b,
 * head h, query block i and each key block j listed in CSR row h_m*nb + i:
 *   E[b][h][i][j] = sum over r in block i with r < n_valid, c in block j with c < n_valid of
 *                   exp(scale * <q_r, k_c> - LSE[b][h][r])
 * where LSE must be the row log-sum-exp over all real keys (what lva_block_sparse_attn
 * returns with the all-ones mask); rows whose LSE is not finite contribute 0.  Key blocks not
 * listed get E = 0, so the whole row E[b][h][i][0..nb) is written.  The sum of a row is the
 * number of real query rows in block i (up to rounding).
 * Arithmetic: bf16 tensor-core products with fp32 accumulation, fp32 exponentials and sums
 * in a fixed order (the result does not depend on timing).
 *
 * q, k: device bf16 [B, H, n_pad, d], 16-byte aligned; lse: device fp32 [B, H, n_pad];
 * energy: device fp32 [B, H, nb, nb] (caller-owned, written).  row_ptr / col_idx / col_len /
 * mask_heads: a CSR block list as for lva_block_sparse_attn (the all-ones list for a dense
 * calibration pass).  Bad CSR rows (outside col_len, a block outside [0, nb), or blocks not
 * strictly ascending) are skipped (their energy row stays 0) and reported through
 * lva_device_error as LVA_ERR_INVALID_ARG.
 * Supported: d in {64, 128}, block_size in {64, 128}, B*H*n_pad < 2^31.
 */
lva_status lva_block_energy(const void* q, const void* k, const float* lse, float* energy, int B,
                            int H, int64_t n_pad, int64_t n_valid, int d, int block_size,
                            const int32_t* row_ptr, const int32_t* col_idx, int64_t col_len,
                            int mask_heads, float scale, cudaStream_t stream);

/*
 * lva_select_blocks -- fewest key blocks reaching a cumulative energy threshold.
 *
 * CalibAtt page (section 2 A.1): for every query block, the minimum number of key blocks
 * needed to reach the cumulative energy threshold eps(t) is selected (eps is higher early in
 * denoising and lower late; the caller passes the value for the timestep).  For every row
 * x of energy[rows][nb]:
 *   order  = key blocks by descending energy, equal energies by ascending index;
 *   S_k    = sum of the first k energies of that order, one float64 addition at a time;
 *   k*     = the smallest k >= 0 with S_k >= eps * S_nb (float64 product);
 *   mask[x][j] = 1 for the first k* blocks of the order, else 0.
 * A row of zeros (a query block of padding rows) selects nothing; eps = 0 selects nothing.
 *
 * energy: device fp32 [rows, nb], finite and >= 0 (a row holding anything else selects
 * nothing and is reported through lva_device_error as LVA_ERR_INVALID_ARG, detail = row).
 * mask: device uint8 [rows, nb] (caller-owned, written).  eps in [0, 1].
 * Supported: 1 <= nb <= 4096 (LVA_ERR_UNSUPPORTED beyond).
 */
lva_status lva_select_blocks(const float* energy, uint8_t* mask, int64_t rows, int nb, double eps,
                             cudaStream_t stream);

/*
 * lva_aggregate_masks -- cross-prompt agreement of calibration masks.
 *
 * CalibAtt page (section 2 A.2): the masks of the calibration prompts are averaged and a
 * block is kept only when it was selected in a large enough fraction rho of them, which gives
 * one data-independent mask per (timestep, layer, head).  For x < count:
 *   out[x] = 1 if (number of p < prompts with masks[p*count + x] != 0) >= rho * prompts
 *            (compared in float64), else 0.
 * masks: device uint8 [prompts, count]; out: device uint8 [count] (caller-owned, written).
 * prompts >= 1, rho in [0, 1].  The result is the dense input of the STATIC mask kind.
 */
lva_status lva_aggregate_masks(const uint8_t* masks, uint8_t* out, int prompts, int64_t count,
                               double rho, cudaStream_t stream);

/* Shape of one attention layer over a T x Hg x Wg latent grid (lva_layer_step_host). */
typedef struct {
  int B, H;                    /* batch elements and heads */
  int d;                       /* head dim: 64 or 128 */
  int block_size;              /* 64 or 128 */
  int T, Hg, Wg;               /* latent grid: N = T*Hg*Wg tokens */
  int tile_t, tile_h, tile_w;  /* tiles of the token order (lva_reorder_tokens) */
  float scale;                 /* softmax scale, e.g. 1/sqrt(d) */
} lva_layer_shape;

/* Device buffers and events of lva_layer_step_host, all owned by the caller.  With
 * n_pad = N rounded up to block_size and nb = n_pad / block_size: */
typedef struct {
  void* qkv_stage;      /* device bf16 [3, B, H, N, d]: the step's raster Q, K, V */
  void* o_stage;        /* device bf16 [B, H, N, d]: the step's raster O */
  float* lse_stage;     /* device fp32 [B, H, n_pad]: the step's LSE (tile order) */
  void* qkv_tile;       /* device bf16 [3, B, H, n_pad, d]: Q, K, V in tile order */
  void* o_tile;         /* device bf16 [B, H, n_pad, d]: O in tile order; only with query_src */
  int32_t* row_ptr;     /* device int32 [mask_heads*nb + 1] */
  int32_t* col_idx;     /* device int32 [col_capacity] */
  int64_t col_capacity;
  int64_t col_len;      /* CSR entries the attention may read: col_capacity, or the exact entry
                           count when known (short rows then run several blocks per CTA) */
  int32_t* nnz;         /* device int32 [1] */
  cudaEvent_t* events;  /* num_events caller-created events, at least 2*groups + 2 */
  int num_events;
} lva_host_step_buffers;

/*
 * lva_layer_step_host -- one attention layer from and to pinned host memory.
 *
 * The layer step of the LVSA page ("LVSA: Training-Free Sparse Attention for Long Video
 * Diffusion", technical summary section 2) and of the CalibAtt page ("Accelerating
 * Text-to-Video Generation with Calibrated Sparse Attention", section 2 B) for inputs that
 * live in host memory: for every batch element and group of heads,
 *   copy raster Q, K, V in -> lva_reorder_tokens -> lva_block_sparse_attn_raster -> copy O
 *   and LSE out,
 * with the CSR of the step's mask built once first (lva_build_block_mask with `mask`, when
 * build_mask != 0; otherwise row_ptr / col_idx must already hold it).  With query_src (the
 * repetitive heads of lva_block_sparse_attn) a group runs lva_block_sparse_attn into o_tile,
 * lva_broadcast_blocks and the inverse lva_reorder_tokens instead.  The results are those
 * of the same calls on device buffers, bit for bit.
 *
 * Heads are split into up to ceil(head_groups / B) groups per batch element (runs of
 * ceil(H / groups) heads).  Each group's three input copies (one cudaMemcpyAsync each) go on
 * `h2d`, its compute on `compute` and its two output copies on `d2h`, ordered by the events
 * of `bufs`, so one group's copies overlap the others' compute.  Two buffer sets (each with
 * its own staging, outputs and events; the tile-order and CSR buffers may be shared) used
 * alternately let consecutive steps overlap as well: a step waits only for the previous use
 * of its own buffer set.
 *
 * qkv_host: pinned bf16 [3, B, H, N, d] raster Q, K, V (read); o_host: pinned bf16
 * [B, H, N, d] raster O (written); lse_host: pinned fp32 [B, H, n_pad] tile-order LSE
 * (written).  mask: n_valid = N, n_pad and block_size as the shape gives them, step inside;
 * dense_mask: device, STATIC only.  *done (may be NULL) receives the event of `bufs` that
 * completes once o_host and lse_host hold the results; until then the host buffers must not
 * be touched.  Returns after enqueueing; nothing is allocated.
 * Errors: LVA_ERR_INVALID_ARG for bad shapes, null or unpinned buffers, too few events;
 * LVA_ERR_UNSUPPORTED for a head dim or block size without a kernel; LVA_ERR_CAPACITY when
 * col_capacity is below lva_block_mask_max_nnz; all before anything is enqueued.  Errors of
 * the enqueued calls are returned as they occur (work already enqueued stays enqueued).
 */
lva_status lva_layer_step_host(const void* qkv_host, void* o_host, float* lse_host,
                               const lva_layer_shape* shape, const lva_mask_params* mask,
                               const uint8_t* dense_mask, int build_mask, const int32_t* query_src,
                               int src_heads, const lva_host_step_buffers* bufs, int head_groups,
                               cudaStream_t compute, cudaStream_t h2d, cudaStream_t d2h,
                               cudaEvent_t* done);

/*
 * lva_device_error -- read and clear the current device's kernel error word.
 *
 * Synchronises `stream`, then stores in *status the first kernel-side fault recorded since
 * the last call (LVA_OK if none): LVA_ERR_INVALID_ARG for CSR entries out of range,
 * LVA_ERR_TIMEOUT for a pipeline wait that ran past its limit.  *detail (may be NULL)
 * receives a kernel-specific code locating the fault.  The word is taken and cleared in one
 * atomic step on `stream`: a fault that a kernel on another stream records meanwhile is
 * reported by this call or the next, never lost.  Concurrent calls on one device are
 * serialised.
 */
lva_status lva_device_error(cudaStream_t stream, lva_status* status, int* detail);

/*
 * lva_selftest_wait -- diagnostic of the kernels' bounded waits; the pages have no counterpart.
 *
 * Every pipeline wait in these kernels (TMA arrivals, MMA completions, softmax hand-offs)
 * polls its mbarrier for at most 2 s of device wall time (%globaltimer), or until another role
 * of the same CTA raises the CTA's abort flag, then gives up and records LVA_ERR_TIMEOUT in
 * the device error word, so a broken pipeline ends with a status instead of a hung GPU.  This
 * call runs that same wait in a one-CTA kernel on `stream`:
 *   mode 0: nothing arrives; after about 2 s the error word holds (LVA_ERR_TIMEOUT, 100);
 *   mode 1: a second warp raises the abort flag after about 1 ms;
 *           the error word holds (LVA_ERR_TIMEOUT, 101);
 *   mode 2: a second warp arrives after about 1 ms; the wait completes, nothing is recorded.
 * Read the outcome with lva_device_error.  The kernel touches no caller memory; the context
 * stays usable in every mode.  Returns LVA_ERR_INVALID_ARG for another mode.
 */
lva_status lva_selftest_wait(int mode, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LVA_H */

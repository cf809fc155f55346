/*
 * svg.h -- C ABI of the B200 (sm_100a) sparse spatial/temporal video attention
 * library.
 *
 * The library implements one attention layer of Sparse VideoGen-style sparse
 * 3D attention for video diffusion transformers:
 *
 *   0. svg_qk_norm_rope         (optional) QK-Norm + RoPE of q and k, with
 *                               their token-major copies in the same pass;
 *   1. svg_profile_heads        online profiling: per head, pick the spatial or
 *                               the temporal mask from a few sampled queries;
 *   2. svg_permute_token_major  frame-major -> token-major reordering of the
 *                               heads that run temporal
 *                               (svg_permute_temporal_heads: those heads only,
 *                               the copy the fused attention reads);
 *   3. svg_build_block_mask     per-query-block key-block lists (CSR) from the
 *                               spatial / temporal geometry, or
 *      svg_block_energy +
 *      svg_build_block_mask_calibrated   lists from cumulative-energy calibration
 *                               (svg_epsilon_schedule, svg_lists_to_intervals,
 *                               svg_lists_to_bitmap: schedule and encodings);
 *   4. svg_sparse_attn          block-sparse attention over 128x128 tiles that
 *                               walks only the kept key blocks
 *                               (svg_sparse_attn_fused: with the reordering of
 *                               temporal heads folded in; svg_v_exponents:
 *                               per-head V scale for its fp16 P.V;
 *                               svg_pair_query_tiles: a pairing order of the
 *                               query tiles for lists used many times);
 *   5. svg_permute_frame_major  the inverse reordering of the output;
 *   6. svg_row_similarity, svg_anchor_lists, svg_anchor_list_ids,
 *      svg_row_broadcast        spatial-repetition heads (anchor rows only).
 *
 * Sources (cited by page title and section):
 *   [SVG]  Sparse VideoGen article, m.jxzklqfsx.com/article/815093.html
 *   [CAL]  CalibAtt article, lpnh.cn/news/568491
 *   [SURV] video-diffusion acceleration survey, wmrh.cn/news/48564
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  * Tensors q, k, v, o, x, y are caller-owned DEVICE memory, contiguous
 *    row-major [B, H, N, d] with d in {64, 128}; element type per `dtype`
 *    (SVG_BF16 or SVG_FP32).  Base pointers must be 16-byte aligned.
 *  * Tokens are frame-major unless stated: n = f * P + s, where f < F is the
 *    frame, s < P the spatial position and P = tokens_per_frame, N = F * P.
 *    Token-major order is m = s * F + f.
 *  * Tiles are T = 128 tokens; tile i holds tokens [128 i, min(N, 128 i + 128)).
 *    nB = ceil(N / 128).
 *  * The library allocates no device memory.  Scratch it needs is passed in
 *    as `workspace` (device, 256-byte aligned, size from the matching
 *    *_workspace_size call).
 *  * `stream` is a cudaStream_t cast to void*; NULL means the legacy default
 *    stream.  Every call is asynchronous on that stream.  Arguments are
 *    validated on the host before anything is launched; on a non-SVG_OK
 *    return nothing was launched (except SVG_ERR_CUDA, which reports a launch
 *    failure) and svg_last_error() describes the problem.
 *  * Device-side index checks never fault: out-of-range list entries are
 *    skipped and recorded in the optional `device_status` word.
 *  * No call blocks the host, throws, or traps on the device.
 */
#ifndef SVG_B200_H_
#define SVG_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVG_OK = 0,
  SVG_ERR_INVALID_ARG = 1, /* bad shape, pointer, alignment or enum value */
  SVG_ERR_UNSUPPORTED = 2, /* valid request this build does not implement */
  SVG_ERR_CUDA = 3,        /* a CUDA launch or query failed */
  SVG_ERR_TIMEOUT = 4      /* device status: a bounded wait gave up */
} svg_status;

typedef enum { SVG_BF16 = 0, SVG_FP32 = 1 } svg_dtype;

/* Per-head attention mode.  Also the list id svg_sparse_attn uses when the
 * lists are the three geometric ones concatenated in this order. */
typedef enum {
  SVG_MODE_SPATIAL = 0,  /* [SVG] "Spatial Head": same and adjacent frames */
  SVG_MODE_TEMPORAL = 1, /* [SVG] "Temporal Head": same position, all frames */
  SVG_MODE_DENSE = 2     /* every key (only by explicit caller choice) */
} svg_mode;

/* Bits of the optional device status word (int32, device memory, OR-ed). */
#define SVG_DEVICE_BAD_LIST_ID 0x1   /* a list id outside [0, n_lists)      */
#define SVG_DEVICE_BAD_INDEX 0x2     /* a key-block index outside [0, nB)   */
#define SVG_DEVICE_TIMEOUT 0x4       /* a bounded pipeline wait gave up      */
#define SVG_DEVICE_CAPACITY 0x8      /* a list did not fit the given buffer */
#define SVG_DEVICE_RANGE 0x10        /* a V value stayed outside the fp16 range (see 4a) */

#define SVG_TILE 128

/* Layout bits of svg_sparse_attn_fused (section 4b). */
#define SVG_FUSE_INPUT 0x1   /* q, k, v frame-major; temporal heads gathered  */
#define SVG_FUSE_OUTPUT 0x2  /* o written frame-major for temporal heads      */

/* Operation bits of svg_qk_norm_rope (section 2b). */
#define SVG_QK_NORM 0x1  /* RMS-normalise each row over d, times gamma       */
#define SVG_QK_ROPE 0x2  /* rotate channel pairs (2i, 2i+1) by cos / sin    */

/* Library identification, e.g. "svg_b200 0.1 sm_100a". */
const char* svg_version(void);

/* Text of the last error returned on the calling host thread ("" if none). */
const char* svg_last_error(void);

/* Bounded device waits.  Every mbarrier wait of the tcgen05 attention kernel
 * polls at most `polls` times (default 1 << 22, which no working pipeline
 * comes near) before it gives up: the kernel then sets SVG_DEVICE_TIMEOUT in
 * the call's device status word, lets its copies and tensor-core operations
 * in flight finish, frees its tensor memory and returns, so the CUDA context
 * stays usable.  This setting exists to test that path and to diagnose
 * stalls; it is process-wide, applies to launches made after the call, and
 * 0 restores the default.  The pages have no counterpart to it.
 * svg_get_wait_limit returns the current value. */
svg_status svg_set_wait_limit(uint32_t polls);
uint32_t svg_get_wait_limit(void);

/* --------------------------------------------------------------------------
 * 1. Online head profiling
 *    [SVG] section "動態自適應的稀疏策略", steps 1-3: sample a few query
 *    tokens, compute their attention under the spatial and the temporal
 *    masks, compare each with dense attention, and give every head the mask
 *    of smaller error.
 *
 *  q, k, v       device [B, H, N, d], frame-major.
 *  sample_idx    device int32 [S], frame-major token indices in [0, N),
 *                shared by every (b, h).  1 <= S <= 64.  Values outside
 *                [0, N) are clamped into range on the device.
 *  frames, tokens_per_frame   F and P with F * P == N.
 *  spatial_width w: the spatial mask keeps keys with |f - f'| <= w.
 *                The temporal mask keeps keys with the same position s.
 *  mse_out       device float [B*H][2] or NULL: mean over the S x d sampled
 *                outputs of (o_spatial - o_dense)^2 and (o_temporal - o_dense)^2.
 *  mode_out      device int32 [B*H]: SVG_MODE_TEMPORAL if the temporal error
 *                is strictly smaller, else SVG_MODE_SPATIAL.
 *  workspace     device scratch of svg_profile_workspace_size(...) bytes.
 * Arithmetic: bf16 inputs use bf16 tensor-core products with fp32
 * accumulation; fp32 inputs use fp32 arithmetic throughout.  Error sums and
 * the mode decision are fp32.
 * ------------------------------------------------------------------------ */
size_t svg_profile_workspace_size(int B, int H, int N, int d, int S);

svg_status svg_profile_heads(const void* q, const void* k, const void* v, int dtype,
                             int B, int H, int N, int d,
                             int frames, int tokens_per_frame, int spatial_width,
                             const int32_t* sample_idx, int S,
                             float* mse_out, int32_t* mode_out,
                             void* workspace, size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------------
 * 1b. Online head profiling without caller-provided scratch
 *    The pages have no counterpart to this entry point; it exists for callers
 *    that cannot allocate device memory (a plugin inside an engine that owns
 *    all device memory and passes no workspace, or a region of a program
 *    where a cudaMalloc would synchronise the device or is not allowed).
 *
 *  Same arguments and results as svg_profile_heads, minus the workspace: the
 *  scratch is a 16 MiB array in device global memory owned by the library
 *  (every GPU that loads the library holds it until the process exits).
 *  The keys of each head are cut into fewer, longer ranges when needed so
 *  that the states fit; results agree with svg_profile_heads to rounding.
 *  Limit: the states of one key range plus the per-row error sums,
 *  B*H*(2*64*(d+2)*4 + 512) bytes, must fit in 16 MiB - 256, i.e.
 *  B*H <= 489 at d = 64 and B*H <= 250 at d = 128; larger shapes return
 *  SVG_ERR_INVALID_ARG.
 *  No device memory is allocated or freed by this call.
 *  The first call on a device looks up the array's device address
 *  (cudaGetSymbolAddress); make that first call on each device before any
 *  stream capture.  The address is kept for the life of the process, so a
 *  cudaDeviceReset (or any teardown of the device's primary context) makes
 *  it stale: do not call this entry point on a device after resetting it.
 *  Every call shares the one array and leaves its contents behind; nothing
 *  in it needs to start at zero.  Calls whose kernels overlap on the GPU
 *  (e.g. on two streams) race on the array: serialise them.
 * ------------------------------------------------------------------------ */
svg_status svg_profile_heads_noalloc(const void* q, const void* k, const void* v, int dtype,
                                     int B, int H, int N, int d,
                                     int frames, int tokens_per_frame, int spatial_width,
                                     const int32_t* sample_idx, int S,
                                     float* mse_out, int32_t* mode_out, void* stream);

/* --------------------------------------------------------------------------
 * 2. / 5. Frame-major <-> token-major permutation
 *    [SVG] section "Layout Transformation + Kernel 加速": reorder so that the
 *    tokens a temporal head needs (one position in every frame) are
 *    contiguous.
 *
 *  svg_permute_token_major:  y[b,h, s*F + f, :] = x[b,h, f*P + s, :]
 *  svg_permute_frame_major:  y[b,h, f*P + s, :] = x[b,h, s*F + f, :]
 *  for every head whose mode[b*H + h] == SVG_MODE_TEMPORAL; every other head
 *  is copied unchanged, so y is always a complete tensor.  mode == NULL
 *  permutes every head.  x and y are device [B, H, N, d] and must not
 *  overlap (out of place).  Bit-exact: pure data movement.
 * ------------------------------------------------------------------------ */
svg_status svg_permute_token_major(const void* x, void* y, int dtype,
                                   int B, int H, int N, int d,
                                   int frames, int tokens_per_frame,
                                   const int32_t* mode, void* stream);

svg_status svg_permute_frame_major(const void* x, void* y, int dtype,
                                   int B, int H, int N, int d,
                                   int frames, int tokens_per_frame,
                                   const int32_t* mode, void* stream);

/*  svg_permute_temporal_heads: the token-major reordering of
 *  svg_permute_token_major for the heads whose mode is SVG_MODE_TEMPORAL
 *  only; every other head of y is left as it is (not written).  This is the
 *  copy svg_sparse_attn_fused reads for temporal heads (q_tm, k_tm, v_tm),
 *  made after profiling at the cost of the temporal heads alone.  mode is
 *  required (NULL: SVG_ERR_INVALID_ARG); other arguments and errors as for
 *  svg_permute_token_major.  Bit-exact. */
svg_status svg_permute_temporal_heads(const void* x, void* y, int dtype,
                                      int B, int H, int N, int d,
                                      int frames, int tokens_per_frame,
                                      const int32_t* mode, void* stream);

/* --------------------------------------------------------------------------
 * 2b. QK-Norm + RoPE of q and k, with optional token-major copies
 *    [SVG] section "Layout Transformation + Kernel 加速": next to the
 *    attention kernels the method ships its own QK-Norm and RoPE kernels.
 *    The pages give no formulas; this call reads them as
 *      QK-Norm: x_hat = x / sqrt(mean_c x_c^2 + eps) * gamma over the d
 *               channels of each (b, h, n) row;
 *      RoPE:    channel pair (2i, 2i+1) = (a, b) of row n becomes
 *               (a cos[n][i] - b sin[n][i], a sin[n][i] + b cos[n][i]);
 *    with the norm first.  One pass reads q and k once and writes the
 *    results frame-major and, when asked, token-major (every head), which
 *    is the reordering the temporal heads need.
 *
 *  q, k          device [B, H, N, d] inputs, frame-major.
 *  q_out, k_out  device [B, H, N, d] results, frame-major.  q_out may be q
 *                itself and k_out k itself (in place); no other overlap.
 *  q_tm_out, k_tm_out  device [B, H, N, d] token-major copies of the
 *                results (row m = s * F + f holds token n = f * P + s), or
 *                both NULL.  When given, frames * tokens_per_frame == N;
 *                otherwise frames and tokens_per_frame are ignored.
 *  ops           SVG_QK_NORM | SVG_QK_ROPE (either, both, or 0 for a copy).
 *  gamma_q, gamma_k  device float [d] per-channel weights, or NULL for 1.
 *  eps           added to the mean square inside the square root; finite,
 *                >= 0 (eps = 0 turns an all-zero row into NaN).
 *  rope_cos, rope_sin  device float [N][d/2] (pair i of token n), required
 *                with SVG_QK_ROPE.
 * Every pointer is 16-byte aligned.  Arithmetic in fp32 (row sums of squares
 * in fp32, reciprocal square root), results rounded to the tensor dtype
 * (bf16: to nearest even).  Bytes: reads 2 B H N d elt, writes 2 or 4 times
 * that, plus the tables once per group of heads.
 * ------------------------------------------------------------------------ */
svg_status svg_qk_norm_rope(const void* q, const void* k, void* q_out, void* k_out,
                            void* q_tm_out, void* k_tm_out, int dtype,
                            int B, int H, int N, int d,
                            int frames, int tokens_per_frame, int ops,
                            const float* gamma_q, const float* gamma_k, float eps,
                            const float* rope_cos, const float* rope_sin, void* stream);

/* --------------------------------------------------------------------------
 * 3a. Geometric key-block lists
 *    [CAL] section 2.2 (keep/skip decisions on 128x128 tiles) applied to the
 *    [SVG] head masks.  Tile pair (i, j) is kept iff some token of query tile
 *    i and some token of key tile j satisfy the token mask:
 *      SVG_MODE_SPATIAL   frame-major tokens, |f - f'| <= spatial_width;
 *      SVG_MODE_TEMPORAL  token-major tokens (the order temporal heads run
 *                         in), same position s;
 *      SVG_MODE_DENSE     every pair.
 *
 *  indptr    device int32 [nB + 1]: row i is indices[indptr[i] - index_base ..
 *            indptr[i+1] - index_base), i.e. every indptr value is offset by
 *            `index_base` (>= 0) so that several lists can share one indices
 *            buffer: pass indices + index_base for a list stored there.
 *  indices   device int32 [capacity], ascending within a row.
 *  nnz_out   device int64 [1]: number of entries.  If it exceeds `capacity`
 *            the indices are not written (indptr and nnz still are) and
 *            SVG_DEVICE_CAPACITY is set in *device_status (if non-NULL).
 *            capacity = nB * nB always suffices.
 * ------------------------------------------------------------------------ */
svg_status svg_build_block_mask(int kind, int frames, int tokens_per_frame,
                                int spatial_width, int N,
                                int32_t* indptr, int32_t* indices, int64_t capacity,
                                int64_t index_base, int64_t* nnz_out,
                                int32_t* device_status, void* stream);

/* --------------------------------------------------------------------------
 * 3b. Block energy for calibration
 *    [CAL] section 3.1: the attention energy E(r, c) of query block r on key
 *    block c.  E[b,h,r,c] = sum over rows i of block r and keys j of block c
 *    of softmax_j(q_i . k_j / sqrt(d)), divided by the row count of block r,
 *    so every row of E sums to 1.
 *
 *  q, k      device [B, H, N, d].
 *  energy    device float [B*H][nB][nB].
 *  workspace device scratch of svg_block_energy_workspace_size(...) bytes.
 * ------------------------------------------------------------------------ */
size_t svg_block_energy_workspace_size(int B, int H, int N);

svg_status svg_block_energy(const void* q, const void* k, int dtype,
                            int B, int H, int N, int d, float* energy,
                            void* workspace, size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------------
 * 3c. Calibrated key-block lists
 *    [CAL] section 3.1: for every list l, input r and query block i, sort the
 *    key blocks by descending energy (ties: smaller index first) and keep the
 *    shortest prefix whose running sum (float64, in that order) reaches eps;
 *    over the R inputs keep block c iff (#inputs keeping c) / R >= rho
 *    (float64); a row left empty keeps the block of largest summed energy
 *    (float64 sum over inputs in order; smallest index on ties).
 *
 *  energy    device float [R][L][nQB][nKB] (e.g. svg_block_energy outputs for
 *            R inputs, with L = B*H lists).  1 <= R <= 16, nKB <= 4096.
 *  indptr    device int32 [L][nQB + 1], offsets into the shared `indices`
 *            (list l row i: indices[indptr[l*(nQB+1)+i] .. indptr[l*(nQB+1)+i+1])).
 *  indices   device int32 [capacity]; nnz_out, device_status as in 3a.
 *            capacity = L * nQB * nKB always suffices.
 *  workspace device scratch of svg_calibrated_workspace_size(...) bytes.
 * Given the same energies, the lists are bit-identical to a float64
 * evaluation of the rule above (the running sums use the same order).
 * ------------------------------------------------------------------------ */
size_t svg_calibrated_workspace_size(int L, int nQB, int nKB);

svg_status svg_build_block_mask_calibrated(const float* energy, int R, int L,
                                           int nQB, int nKB, double eps, double rho,
                                           int32_t* indptr, int32_t* indices,
                                           int64_t capacity, int64_t* nnz_out,
                                           int32_t* device_status,
                                           void* workspace, size_t workspace_bytes,
                                           void* stream);

/* --------------------------------------------------------------------------
 * 3c. Threshold schedule and mask encodings
 *    [CAL] section 3.1: the energy threshold eps(t) of the calibration decays
 *    exponentially over the denoising steps, about 0.99 at the first and
 *    0.84 at the last; section 3.3: the sparse mask is precomputed as a skip
 *    list of contiguous block intervals and stored as a bitmap (32x less
 *    memory than one 32-bit value per block pair).
 *
 *  svg_epsilon_schedule (host only, no device work):
 *    eps_out[i] = eps_first * (eps_last / eps_first)^(i / (n_steps - 1)),
 *    i in [0, n_steps); one step gives eps_first.  eps_out is a HOST array of
 *    n_steps doubles; thresholds must lie in (0, 1].  Feed eps_out[t] to
 *    svg_build_block_mask_calibrated for the lists of step t.
 *
 *  svg_lists_to_intervals:
 *    indptr / indices  device CSR of n_rows rows over n_cols key blocks,
 *                      indices ascending within a row (duplicates allowed);
 *    iptr     device int32 [n_rows + 1]: row r's runs are
 *             [iptr[r], iptr[r + 1]) of starts / ends;
 *    starts, ends  device int32 [capacity]: maximal runs of consecutive kept
 *             blocks, half-open [start, end), ascending;
 *    n_out    device int64: total runs (written in every case);
 *    capacity 0 is a size query (only iptr and n_out are written).
 *    Indices outside [0, n_cols) or a descending row set
 *    SVG_DEVICE_BAD_INDEX (the row's runs are then unspecified); runs past
 *    capacity are dropped and set SVG_DEVICE_CAPACITY.
 *
 *  svg_lists_to_bitmap:
 *    bitmap   device uint32 [n_rows][ceil(n_cols / 32)]: block c of row r is
 *             bit (c mod 32) of word (c div 32); every word is written.
 *    Indices outside [0, n_cols) are skipped and set SVG_DEVICE_BAD_INDEX.
 * Integer work: bit-exact.
 * ------------------------------------------------------------------------ */
svg_status svg_epsilon_schedule(int n_steps, double eps_first, double eps_last, double* eps_out);

svg_status svg_lists_to_intervals(int n_rows, int n_cols, const int32_t* indptr,
                                  const int32_t* indices, int32_t* iptr, int32_t* starts,
                                  int32_t* ends, int64_t capacity, int64_t* n_out,
                                  int32_t* device_status, void* stream);

svg_status svg_lists_to_bitmap(int n_rows, int n_cols, const int32_t* indptr,
                               const int32_t* indices, uint32_t* bitmap, int32_t* device_status,
                               void* stream);

/* --------------------------------------------------------------------------
 * 4. Block-sparse attention
 *    [SURV] section 2.1 (softmax(Q K^T / sqrt(d)) V), [CAL] sections 2.2 and
 *    3.3 (128x128 tiles, per-query-block list of kept key blocks).  For every
 *    (b, h) and query tile i, with l = list_id[b*H + h]:
 *        o[rows of tile i] = softmax over every key j < N of every kept tile
 *                            (scale * q . k_j) . v_j
 *    A kept tile is attended in full; a query tile with an empty list gets
 *    o = 0.  Heads that run temporal pass token-major q/k/v and get
 *    token-major o (see svg_permute_*).
 *
 *  q, k, v, o   device [B, H, N, d]; o may not alias q, k or v.
 *  list_id      device int32 [B*H] in [0, n_lists).  With the three
 *               geometric lists concatenated as (spatial, temporal, dense),
 *               the profiling output mode_out is a valid list_id.
 *  indptr       device int32 [n_lists][n_qblocks + 1], absolute offsets into
 *               `indices`; n_qblocks must equal nB.
 *  indices      device int32, key-block indices in [0, nB), strictly
 *               ascending per row (a row is a set of key blocks).  An entry
 *               outside [0, nB), or not above the row's previous used entry
 *               (a repeat or a descending entry), is skipped and sets
 *               SVG_DEVICE_BAD_INDEX; no key block is attended twice.
 *  scale        softmax scale; 0 selects 1/sqrt(d).
 *  device_status  optional device int32 (may be NULL), see SVG_DEVICE_*.
 *  v_exp        optional device int32 [B*H] from svg_v_exponents (may be
 *               NULL: every exponent 0).  Head (b, h) converts v * 2^-e to
 *               fp16 and multiplies its output by 2^e, exactly (powers of
 *               two), so any finite bf16 V gives the right result.
 * Arithmetic (bf16): Q.K^T on bf16 tensor cores with fp32 accumulation, fp32
 * online softmax; P.V on fp16 tensor cores (P in [0, 256] with an 11-bit
 * significand; V converted from bf16 to fp16 on chip, exact for
 * |v| * 2^-e <= 65504) with fp32 accumulation; output rounded to nearest
 * bf16.  A visited V value that stays beyond the fp16 range (no v_exp given,
 * or an inf / NaN) becomes inf and sets SVG_DEVICE_RANGE.  fp32 inputs use
 * fp32 arithmetic throughout and ignore v_exp.
 * ------------------------------------------------------------------------ */
svg_status svg_sparse_attn(const void* q, const void* k, const void* v, void* o, int dtype,
                           int B, int H, int N, int d,
                           const int32_t* list_id, int n_lists, int n_qblocks,
                           const int32_t* indptr, const int32_t* indices,
                           float scale, int32_t* device_status, const int32_t* v_exp,
                           void* stream);

/* --------------------------------------------------------------------------
 * 4a. V exponents for the fp16 P.V product
 *    The pages have no counterpart: it keeps the tensor-core arithmetic of
 *    section 4 exact in range for every finite bf16 V.  For every (b, h):
 *        exps[b*H + h] = the smallest e >= 0 with max |v[b,h]| * 2^-e <= 65504
 *    (0 when the head already fits fp16; 255 when it holds inf or NaN).  One
 *    read of v.  bf16 only.
 *
 *  v      device bf16 [B, H, N, d], 16-byte aligned.
 *  exps   device int32 [B*H] (written; zeroed by this call first).
 * ------------------------------------------------------------------------ */
svg_status svg_v_exponents(const void* v, int dtype, int B, int H, int N, int d, int32_t* exps,
                           void* stream);

/* --------------------------------------------------------------------------
 * 4b. Block-sparse attention with the layout transformation fused in
 *    [SVG] sections "Temporal Head" and "Layout Transformation + Kernel 加速":
 *    temporal heads attend in token-major order (a token's keys across frames
 *    are contiguous there).  With layout = SVG_FUSE_INPUT | SVG_FUSE_OUTPUT,
 *    svg_sparse_attn_fused computes exactly
 *        x' = svg_permute_token_major(x, mode) for x in q, k, v
 *        o' = svg_sparse_attn(q', k', v', list_id = mode)
 *        o  = svg_permute_frame_major(o', mode)
 *    without the intermediate tensors.  Each side can be fused on its own:
 *      SVG_FUSE_INPUT   q, k, v are FRAME-MAJOR for every head; heads with
 *                       mode == SVG_MODE_TEMPORAL gather their rows in
 *                       token-major order (otherwise such heads' q, k, v are
 *                       already token-major, e.g. from svg_permute_token_major);
 *      SVG_FUSE_OUTPUT  o is written FRAME-MAJOR for every head (otherwise
 *                       temporal heads' o is token-major).
 *    layout 0 is svg_sparse_attn with list_id = mode.
 *    Token-major copies: q_tm, k_tm, v_tm (all three or none; not with
 *    SVG_FUSE_INPUT) hold every head in token-major order, e.g. from
 *    svg_permute_token_major with mode NULL; temporal heads read them and the
 *    other heads read q, k, v (frame-major).  The copies then do not depend
 *    on the modes, so they can be made while the heads are being profiled.
 *
 *  q, k, v, o   device [B, H, N, d] in the layouts above.
 *  q_tm, k_tm, v_tm   device [B, H, N, d] or NULL.
 *  frames, tokens_per_frame   F and P with F * P == N (unused for layout 0).
 *  mode         device int32 [B*H]: the list id of each head (as list_id in
 *               svg_sparse_attn, e.g. the profiling output with the three
 *               geometric lists concatenated) and its token order.
 *  layout       0 or an OR of SVG_FUSE_INPUT and SVG_FUSE_OUTPUT.
 *  tile_order   device int32 [n_lists][n_qblocks] or NULL: per list, the
 *               query tiles in the order the kernel pairs them into work
 *               items (each row a permutation of 0 .. n_qblocks-1, e.g. from
 *               svg_anchor_lists, which puts the tiles with work first).
 *               A scheduling choice only: results do not depend on it.  An
 *               entry outside [0, n_qblocks) is skipped and sets
 *               SVG_DEVICE_BAD_INDEX; a row that is not a permutation leaves
 *               missing tiles unwritten.  fp32 inputs ignore it.
 *  Other arguments, errors and arithmetic as in svg_sparse_attn; a mode
 *  outside [0, n_lists) sets SVG_DEVICE_BAD_LIST_ID and gives o = 0 for the
 *  head.
 * ------------------------------------------------------------------------ */
svg_status svg_sparse_attn_fused(const void* q, const void* k, const void* v,
                                 const void* q_tm, const void* k_tm, const void* v_tm, void* o,
                                 int dtype, int B, int H, int N, int d, int frames,
                                 int tokens_per_frame, const int32_t* mode, int layout,
                                 int n_lists, int n_qblocks, const int32_t* indptr,
                                 const int32_t* indices, const int32_t* tile_order, float scale,
                                 int32_t* device_status, const int32_t* v_exp, void* stream);

/* --------------------------------------------------------------------------
 * 4c. Pairing order of query tiles
 *    [CAL] sections 2.2 and 3.3: attention on 128 x 128 tiles through
 *    per-query-block lists of kept key blocks.  svg_sparse_attn_fused runs
 *    two query tiles of a head as one work item and loads a key block kept
 *    by both once; tile_order says which tiles go together.  This pass
 *    computes, per list, an order in which consecutive pairs share many key
 *    blocks: greedily, the smallest unpaired query tile takes the unpaired
 *    tile whose row has the most key blocks in common with its own (ties:
 *    the smaller index).  A scheduling choice only (results do not depend on
 *    it); meant for lists that are built once and used many times (the
 *    calibrated lists).
 *
 *  indptr       device int32 [n_lists][n_qblocks + 1], absolute offsets into
 *               indices (as for svg_sparse_attn).
 *  indices      device int32 key-block indices; an index outside
 *               [0, n_kblocks) or a bad row range is skipped and sets
 *               SVG_DEVICE_BAD_INDEX in device_status (may be NULL).
 *  tile_order   device int32 [n_lists][n_qblocks], written: each row a
 *               permutation of 0 .. n_qblocks-1, paired as (2i, 2i + 1).
 *  workspace    device, 4-byte aligned, at least
 *               svg_pair_query_tiles_workspace_size(n_lists, n_qblocks,
 *               n_kblocks) bytes (the rows as bitmaps).
 *  Errors: SVG_ERR_INVALID_ARG for null pointers, non-positive sizes, more
 *  than 65535 lists, a short or misaligned workspace, or rows too many for
 *  the pass's shared memory (n_qblocks + (n_kblocks + 31) / 32 * 4 bytes
 *  beyond 48 KB).
 * ------------------------------------------------------------------------ */
size_t svg_pair_query_tiles_workspace_size(int n_lists, int n_qblocks, int n_kblocks);

svg_status svg_pair_query_tiles(const int32_t* indptr, const int32_t* indices, int n_lists,
                                int n_qblocks, int n_kblocks, int32_t* tile_order,
                                int32_t* device_status, void* workspace, size_t workspace_bytes,
                                void* stream);

/* --------------------------------------------------------------------------
 * 6. Spatial-repetition heads
 *    [CAL] section 3.2: in some heads the image rows of a frame attend almost
 *    alike.  They are found by the mean cosine similarity of the rows'
 *    attention patterns (repeating when it exceeds gamma = 0.87, a caller
 *    decision on the returned value); for them only k = 5 equally spaced
 *    anchor rows per frame are computed and every other row takes its
 *    anchor's output.  A frame is `rows` x `cols` tokens (P = rows * cols,
 *    token n = f P + y cols + x).  Anchors: band j holds the rows y with
 *    floor(y k / rows) = j; its anchor is the band's middle row (the upper
 *    of two); every row is an anchor when k >= rows.
 *
 *  svg_row_similarity -- per head, for each evaluated frame the mean over
 *    all row pairs y < y' of cos(A_y, A_y') = <A_y, A_y'> / (|A_y| |A_y'|),
 *    A_y = the cols x N block of dense attention probabilities
 *    softmax(q k^T / sqrt(d)) of row y's tokens over all N keys (Frobenius
 *    products); then the mean over the evaluated frames.
 *      q, k          device [B, H, N, d], frame-major; N = frames*rows*cols.
 *      rows          2 .. 128.
 *      eval_frames   device int32 [n_frames] frame indices, or NULL for
 *                    frames 0 .. n_frames-1.  Out-of-range values are
 *                    clamped and flagged (SVG_DEVICE_BAD_INDEX).
 *      sim_out       device float [B*H].
 *      workspace     device scratch of svg_row_similarity_workspace_size().
 *    Arithmetic (bf16): scores on bf16 tensor cores with fp32 accumulation,
 *    probabilities exp2(t - lse) rounded to fp16 and multiplied on fp16
 *    tensor cores with fp32 accumulation; fp32 inputs: fp32 SIMT.  An
 *    offline step (two dense passes over the evaluated frames' queries).
 *
 *  svg_anchor_lists -- lists for a layer with repeating heads.  Output lists
 *    0 .. n_lists-1 are the input lists; lists n_lists .. 2 n_lists-1 are
 *    copies in which every query tile that holds no anchor-row token has an
 *    empty list (its rows are all filled by svg_row_broadcast).
 *      indptr, indices  input CSR as for svg_sparse_attn (n_qblocks = nB).
 *      list_id, repeat  device int32 [n_heads]: a head with repeat != 0 and
 *                    a list id in [0, n_lists) other than skip_list gets
 *                    list_id + n_lists in list_id_out; others keep theirs.
 *                    repeat may be NULL (no head moves).  skip_list: a list
 *                    id never moved (e.g. SVG_MODE_TEMPORAL, whose heads
 *                    run token-major), or -1.  list_id NULL builds the lists
 *                    (and order) only; svg_anchor_list_ids then maps the ids
 *                    alone, e.g. every step for lists built once.
 *      out_indptr    device int32 [2 n_lists][n_qblocks + 1], absolute.
 *      out_indices   device int32 [capacity]; 2 x the input entries always
 *                    fit.  Entries past capacity are not written
 *                    (SVG_DEVICE_CAPACITY).
 *      list_id_out   device int32 [n_heads].
 *      tile_order_out  device int32 [2 n_lists][n_qblocks] or NULL: per
 *                    output list the pairing order for svg_sparse_attn_fused
 *                    (index order for the first n_lists; for the copies the
 *                    tiles holding anchor rows first, then the others).
 *
 *  svg_row_broadcast -- in place on o [B, H, N, d] (frame-major): for each
 *    head with list_id[b*H+h] >= n_lists (as set by svg_anchor_lists), row
 *    (f, y, x) takes the value of row (f, anchor(y), x); anchor rows and
 *    other heads are untouched.
 * ------------------------------------------------------------------------ */
size_t svg_row_similarity_workspace_size(int dtype, int B, int H, int rows, int cols,
                                         int n_frames);

svg_status svg_row_similarity(const void* q, const void* k, int dtype, int B, int H, int N, int d,
                              int frames, int rows, int cols, const int32_t* eval_frames,
                              int n_frames, float* sim_out, void* workspace,
                              size_t workspace_bytes, int32_t* device_status, void* stream);

svg_status svg_anchor_lists(int n_lists, int n_qblocks, const int32_t* indptr,
                            const int32_t* indices, int N, int frames, int rows, int cols,
                            int anchors, const int32_t* list_id, const int32_t* repeat,
                            int n_heads, int skip_list, int32_t* out_indptr,
                            int32_t* out_indices, int64_t capacity, int32_t* list_id_out,
                            int32_t* tile_order_out, int32_t* device_status, void* stream);

svg_status svg_anchor_list_ids(const int32_t* list_id, const int32_t* repeat, int n_heads,
                               int n_lists, int skip_list, int32_t* list_id_out, void* stream);

svg_status svg_row_broadcast(void* o, int dtype, int B, int H, int N, int d, int frames, int rows,
                             int cols, int anchors, const int32_t* list_id, int n_lists,
                             void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVG_B200_H_ */

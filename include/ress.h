/*
 * ress.h - C ABI of the B200 (sm_100a) block-sparse global attention library.
 *
 * The library implements the hot path shared by the training-free sparse
 * global-attention methods for multi-view 3D transformers (VGGT-style):
 *
 *   1. ress_select_blocks      pooled block selection: mean-pool Q and K per
 *                              block, per-head softmax over pooled logits,
 *                              optional value-contrast term, exact-budget
 *                              top-k per query block (ties to the lower index).
 *   2. ress_block_sparse_attn  attention restricted to the kept key blocks.
 *   3. ress_block_drift        per-dropped-block drift norm and drop-set drift.
 *
 * ress_select_blocks_cdf is the SparseVGGT variant of stage 1: a per-row
 * cumulative probability threshold instead of a fixed budget.
 *
 * Sources: ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers
 * (thelatestinai.com) - Abstract, Fig. 1, Fig. 3, Table 1, Table S5, Table S6;
 * VASC: Value-Aware Sparse Attention with Cross-Layer Memory (paperlayer.ai) -
 * sections 4.1, 4.2, A.1, A.2, A.3.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors are token-major: q, k, v and out are [N][H][d] (d contiguous, one
 *   token row is H*d elements).  lse is [H][N].  idx is [H][nb][budget] int32.
 * - d must be 64.  The block size B (query blocks and key blocks alike) is 64
 *   or 128, and N must be a multiple of B; nb = N / B.  Padding tokens, if
 *   any, are ordinary tokens to the library.
 * - All data pointers are device pointers owned by the caller, on the
 *   current device (the library keeps per-device state, such as its error
 *   flag, and looks it up on the device that is current at the call).
 *   The library never allocates, frees or synchronises; every call is asynchronous and
 *   ordered on `stream` (a cudaStream_t passed as void*, NULL = the legacy
 *   default stream).  Scratch memory comes from the caller's `workspace`,
 *   sized by the matching *_workspace_bytes() query, 256-byte aligned.
 * - Argument checks run on the host before any CUDA call and return
 *   RESS_ERR_INVALID_ARG (bad shape, NULL pointer, budget outside [1, nb],
 *   misaligned pointer), RESS_ERR_UNSUPPORTED (valid but not implemented,
 *   e.g. d != 64) or RESS_ERR_WORKSPACE (workspace too small).  A failed
 *   launch returns RESS_ERR_CUDA.  When N == 0 the call returns RESS_OK and
 *   launches nothing.
 * - Kernels never trap.  A device-side wait that exceeds its time limit, or a
 *   kept-block index outside [0, nb) found in a caller-provided idx (such an
 *   index is skipped), sets a device error flag that ress_check_device_errors()
 *   reports and clears.
 */
#ifndef RESS_H
#define RESS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RESS_OK = 0,
  RESS_ERR_INVALID_ARG = 1,
  RESS_ERR_UNSUPPORTED = 2,
  RESS_ERR_WORKSPACE = 3,
  RESS_ERR_CUDA = 4,
  RESS_ERR_TIMEOUT = 5,
  RESS_ERR_BAD_INDEX = 6
} ress_status;

typedef enum {
  RESS_BF16 = 0, /* bfloat16 q, k, v (and out) */
  RESS_F32 = 1   /* float32 q, k, v (and out); attention and drift stage them to bf16 */
} ress_dtype;

typedef struct {
  int64_t n;        /* N: tokens of all views concatenated (multiple of block) */
  int32_t heads;    /* H: attention heads, 1..64 */
  int32_t head_dim; /* d: must be 64 */
  int32_t block;    /* B: 64 or 128 */
  int32_t dtype;    /* ress_dtype of q, k and v */
} ress_shape;

/*
 * Per-view layout of the concatenated sequence, for the layout-aware entry
 * points (VASC 4.2 and A.5: camera and register queries keep dense
 * attention, key blocks made only of special tokens are always kept, and
 * padding takes no part in pooling or attention).  Every view occupies
 * tokens_per_view consecutive tokens; its positions 0 .. real_tokens - 1
 * carry data and the rest is padding; positions 0 .. special_tokens - 1 are
 * the special (camera, register) tokens.  Requirements: tokens_per_view a
 * multiple of the block size and a divisor of N, 1 <= real_tokens <=
 * tokens_per_view, 0 <= special_tokens <= real_tokens.  A VGGT view is
 * {1408, 1374, 5}: 1 camera + 4 register + 37 x 37 patch tokens, padded to
 * 22 blocks of 64.
 */
typedef struct {
  int32_t tokens_per_view;
  int32_t real_tokens;
  int32_t special_tokens;
} ress_layout;

/* Library version, (major << 16) | minor. */
int ress_version(void);

/* Human-readable name of a status code; never NULL. */
const char* ress_status_string(ress_status status);

/*
 * Workspace bytes that ress_select_blocks needs for `shape` and `lambda`
 * (0 if the shape is invalid).  Layout, each array 256-byte aligned, with
 * nb_pad = nb rounded up to 256:
 *   - lambda == 0, budget < nb <= 2304 (the tensor-core selection):
 *     Qbar [H][nb][64] f32, then the pooled keys split into tf32 high and low
 *     parts Khi, Klo [H][nb_pad][64] f32, the high parts of 128 evenly spaced
 *     sample keys [H][128][64], the key norms [H][nb] f32, one int32 count
 *     (in a 256-byte slot) and a row list [H][nb] int32;
 *   - otherwise (and for ress_select_blocks_cdf): Qbar [H][nb][64],
 *     Kbar^T [H][64][nb_pad], then Vbar [H][nb][64] and contrast [H][nb]
 *     when lambda > 0, all float32.
 * The size returned covers both layouts when lambda == 0.
 */
size_t ress_select_workspace_bytes(const ress_shape* shape, float lambda);

/*
 * Stage 1: pooled block selection (ReSS Table S5, SpargeAttn row: pooled
 * query/key inner products; VASC 4.1: pooled relevance plus neighbouring
 * value contrast; VASC A.2: an exact-capacity binary Top-K mask).
 *
 * For each head h and query block i:
 *   Qbar_i = mean of the B query tokens of block i (same for Kbar_j, Vbar_j),
 *   s_ij   = (Qbar_i . Kbar_j) / sqrt(d),
 *   p_ij   = softmax over all nb key blocks j of s_ij,
 *   c_j    = ||Vbar_j - Vbar_{j-1}||_2 for j >= 1, c_0 = 0,
 *   score  = p_ij + lambda * c_j,
 * and idx[h][i][0..budget) receives the `budget` blocks of largest score in
 * ascending block order; equal scores go to the lower block index.  With
 * lambda == 0 the ranking uses s_ij, which orders the row as p_ij does.
 *
 *   q, k    [N][H][64] of shape->dtype, 16-byte aligned.
 *   v       [N][H][64], read only when lambda > 0 (may be NULL otherwise).
 *   budget  kept key blocks per query block, 1 <= budget <= nb.
 *   lambda  contrast weight, finite and >= 0.
 *   idx     out, [H][nb][budget] int32.
 *   Supported sizes: nb <= 4096.
 */
ress_status ress_select_blocks(const ress_shape* shape, const void* q, const void* k,
                               const void* v, int32_t budget, float lambda, int32_t* idx,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Stage 1 for callers that cannot allocate device memory.  The pages have no
 * counterpart to this entry point; it exists for callers that may not call
 * cudaMalloc or hold a workspace of their own (for example a plugin running
 * inside another framework's allocator, or a loop in which an allocation,
 * which can synchronise the device, is not allowed).
 *
 * Same arguments, checks and result as ress_select_blocks, without the
 * workspace: the scratch lives in one fixed 32 MiB array in device memory
 * that the library owns (H = 16 and nb <= 2,200 fit, with the value
 * contrast).  Every GPU that loads the library holds that array until the
 * process exits.  A problem whose ress_select_workspace_bytes() exceeds
 * 32 MiB is rejected with RESS_ERR_WORKSPACE before anything is launched.
 *
 * - The first call on a device looks up the array's device address (one
 *   cudaGetSymbolAddress with that device current); make that first call
 *   before any stream capture.  The call allocates nothing.
 * - All calls share the one array, and each call overwrites every scratch
 *   value it reads, so nothing needs to start at zero.  Calls that overlap on
 *   the GPU (different streams, or different host threads, on one device)
 *   race on the array and must be ordered by the caller.
 */
ress_status ress_select_blocks_noalloc(const ress_shape* shape, const void* q, const void* k,
                                       const void* v, int32_t budget, float lambda,
                                       int32_t* idx, void* stream);

/*
 * Stage 1 with the cumulative (CDF) threshold of SparseVGGT instead of a fixed
 * budget (ReSS Table S5: with the similarity gate off, selection is a
 * cumulative threshold on pooled query/key inner products; ReSS Table 2, row
 * "+ CDF threshold").  For each head h and query block i, with p_ij the pooled
 * probabilities of ress_select_blocks (lambda = 0), the count is the smallest
 * m >= 1 such that the m blocks of largest p (equal values in index order) sum
 * to at least tau, or nb if the total never reaches tau.
 *
 *   q, k       as for ress_select_blocks (no V: the rule has no contrast term).
 *   tau        0 < tau <= 1.
 *   capacity   1 <= capacity <= nb: the length of every idx row.
 *   counts     out, [H][nb] int32: the count of every row (it may exceed
 *              capacity).
 *   idx        out, [H][nb][capacity] int32: the top min(count, capacity)
 *              blocks of the row in ascending order, then the last of them
 *              repeated to the end of the row, so that idx with
 *              budget = capacity is a valid kept list for
 *              ress_block_sparse_attn (duplicates count once there).
 *   workspace  ress_select_workspace_bytes(shape, 0) bytes, 256-byte aligned.
 *   Supported sizes: nb <= 4096.
 *   The probabilities are float32 and their running sum is exact (fixed point
 *   in units of 2^-40, independent of the summation order), so the result is
 *   deterministic, and a count can differ from an evaluation in float64 only
 *   where the cumulative mass lies within about 1e-6 of tau.
 */
ress_status ress_select_blocks_cdf(const ress_shape* shape, const void* q, const void* k,
                                   float tau, int32_t capacity, int32_t* counts, int32_t* idx,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Stage 1 with a per-view layout (VASC 4.2 and A.5).  As ress_select_blocks
 * with lambda = 0, except that a block's pooled mean is over its valid
 * (non-padding) tokens only, a key block without a valid token (it pools to
 * zero) ranks below every other block, and a key block whose valid tokens are
 * all special ranks above every other block (such blocks are kept first,
 * lowest index first if there are more of them than the budget).
 *
 *   layout     as described at ress_layout.
 *   workspace  ress_select_workspace_bytes(shape, 0) bytes.
 */
ress_status ress_select_blocks_layout(const ress_shape* shape, const ress_layout* layout,
                                      const void* q, const void* k, int32_t budget,
                                      int32_t* idx, void* workspace, size_t workspace_bytes,
                                      void* stream);

/*
 * Workspace bytes of ress_select_blocks_restore (0 if the shape is invalid):
 * Qbar [H][nb][64], Kbar^T [H][64][nb_pad] and Vbar^T [H][64][nb_pad],
 * float32, each 256-byte aligned.
 */
size_t ress_restore_workspace_bytes(const ress_shape* shape);

/*
 * Stage 1 by drift with iterative residual restoration (ReSS Abstract, Fig. 1,
 * Fig. 3(b)-(c), Fig. 7, Table S3), on pooled contributions.  For query block
 * i of head h, key block j contributes c_j = p_ij Vbar_j to the pooled output
 * (p_ij the pooled probabilities of ress_select_blocks).  The drift score is
 * |c_j|; the initial kept set is the `budget` blocks of largest score (ties
 * to the lower index).  Each of up to `rounds` restoration rounds takes the
 * drop set D and T = sum_{j in D} c_j, forms the pairs of the `candidates`
 * dropped blocks of largest 2 <T, c_b> - |c_b|^2 and the `candidates` kept
 * blocks of smallest 2 <T, c_a> + |c_a|^2 (ties to the lower index), and swaps
 * the pair of smallest |T - c_b + c_a| (ties: lower b, then lower a) when
 * that is below |T|; otherwise restoration stops.  The swap rule and the
 * pooled contributions are this library's reading: the pages give neither.
 *
 *   rounds       0 .. 64 (0: the initial set).
 *   candidates   1 .. 16 per side.
 *   idx          out, [H][nb][budget] int32, ascending.
 *   drift_init   out, [H][nb] float32, |sum over the initial drop set|; or NULL.
 *   drift_final  out, [H][nb] float32, the same for the result; or NULL.
 *   Supported sizes: nb <= 4096.  Arithmetic in float32; a decision between
 *   two values equal to float32 rounding may go either way.
 */
ress_status ress_select_blocks_restore(const ress_shape* shape, const void* q, const void* k,
                                       const void* v, int32_t budget, int32_t rounds,
                                       int32_t candidates, int32_t* idx, float* drift_init,
                                       float* drift_final, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * Workspace bytes of ress_select_blocks_vasc (0 if the shape is invalid):
 * Qbar [H][nb][64], Kbar^T and Vbar^T [H][64][nb_pad] float32, then per pair
 * the contrast and the memory's ranking copy (float32), the demand sum
 * (uint64) and the service count (uint32), [H][(nb + 1) / 2] each; every
 * array 256-byte aligned.
 */
size_t ress_vasc_workspace_bytes(const ress_shape* shape);

/*
 * Stage 1 as VASC selects it, one global layer per call: value-aware demand,
 * a binary mask of exactly c_h blocks per row, and the cross-layer memory
 * settled by what was executed (VASC 4.1, 4.2, 4.3, A.1 - A.5; per-head
 * budgets c_h as in ReSS Fig. 3 and Table 2).
 *
 * Key blocks form fixed pairs of neighbours (2p, 2p+1), p < (nb + 1) / 2; an
 * odd final block is a singleton.  For head h and query block i, with p_ij
 * the pooled probabilities of ress_select_blocks:
 *   rho_p  = sqrt( (1/64) sum_d (Vbar_2p,d - Vbar_2p+1,d)^2 ), 0 for a
 *            singleton (the RMS contrast of the pair); 1 for every pair when
 *            value_aware == 0 (the contrast set to one);
 *   a_ij   = min(1, c_h * p_ij rho_pair(j) / sum_j p_ij rho_pair(j))
 *            (0 when the sum is 0): the demand, rescaled to the capacity and
 *            clipped at one;
 *   mhat_p = memory_p / max over the head's pairs (0 when that is 0): the
 *            ranking copy of the memory;
 *   kept   = the c_h largest a_ij + mhat_pair(j), ties to the lower index.
 * Then, with D_p and S_p the means of a_ij and of the kept mask over all query
 * blocks i and the children j of pair p,
 *   memory_p <- max(0, memory_p + D_p - S_p).
 * How the contrast modulates the relevance (a factor), how memory enters the
 * ranking (added), how it is normalised (by the head's largest balance) and
 * the rescaling (proportional, one clip) are this library's readings.
 *
 *   v            [N][H][64], needed when value_aware != 0 (else may be NULL).
 *   budgets      HOST array of H int32: c_h, 1 <= c_h <= capacity.
 *   capacity     1 <= capacity <= nb: the length of every idx row.
 *   value_aware  1: contrast on; 0: contrast one.
 *   reset        1: the memory is taken as zero on entry (the first global
 *                layer of an inference, or a changed layout); 0: carried in.
 *   memory       in/out, device [H][(nb + 1) / 2] float32 (>= 0).
 *   idx          out, [H][nb][capacity] int32: row (h, i) holds its c_h kept
 *                blocks ascending, then the last of them repeated, a valid
 *                kept list for ress_block_sparse_attn with budget = capacity.
 *   demand       out, [H][(nb + 1) / 2] float32, D; or NULL.
 *   service      out, [H][(nb + 1) / 2] float32, S; or NULL.
 *   workspace    ress_vasc_workspace_bytes(shape) bytes, 256-byte aligned.
 *   Supported sizes: nb <= 4096.  The demand sums are exact in fixed point
 *   (units of 2^-32), so memory, demand and service do not depend on the
 *   order of the kernel's blocks; the scores are float32, so a ranking
 *   decision between two values equal to float32 rounding may go either way.
 */
ress_status ress_select_blocks_vasc(const ress_shape* shape, const void* q, const void* k,
                                    const void* v, const int32_t* budgets, int32_t capacity,
                                    int32_t value_aware, int32_t reset, float* memory,
                                    int32_t* idx, float* demand, float* service,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Workspace bytes that ress_block_sparse_attn and ress_block_drift need:
 * 0 for bf16 inputs; 3 * N * H * 64 * 2 for float32 inputs (bf16 copies of
 * q, k and v).
 */
size_t ress_attn_workspace_bytes(const ress_shape* shape);

/*
 * Stage 2: block-sparse attention forward (ReSS Table S6: the selection feeds
 * one shared block-sparse kernel on the block grid; VASC 4.2: the binary mask
 * is passed directly to the sparse kernel; ReSS Table S5: bidirectional, no
 * causal mask).
 *
 * For query token n of block i and head h, with kept set K(h, i) = idx[h][i]:
 *   out[n][h] = sum_{t in K} softmax_t((q[n][h] . k[t][h]) / sqrt(d)) v[t][h],
 * normalised over the kept tokens only, and
 *   lse[h][n] = ln sum_{t in K} exp((q[n][h] . k[t][h]) / sqrt(d)).
 *
 *   idx    [H][nb][budget] int32 device array; rows need not be sorted or
 *          unique (duplicates count once); entries outside [0, nb) are skipped
 *          and flagged (RESS_ERR_BAD_INDEX via ress_check_device_errors).
 *   out        [N][H][64] of `out_dtype` (RESS_BF16 or RESS_F32, independent
 *              of the input dtype).
 *   lse        [H][N] float32, or NULL.
 *   Supported sizes: nb <= 10,000 (the kept-block lists live in shared
 *   memory); larger grids return RESS_ERR_UNSUPPORTED.
 *   The contractions run on bf16 operands with float32 accumulation; the
 *   probabilities enter P V as bf16 and the row normaliser is the sum of those
 *   same bf16 values, so each output row is a convex combination of kept
 *   values, and lse is the log of that same sum (it differs from the float32
 *   log-sum-exp by at most ln(1 + 2^-9) < 2e-3).
 */
ress_status ress_block_sparse_attn(const ress_shape* shape, const void* q, const void* k,
                                   const void* v, int32_t budget, const int32_t* idx,
                                   void* out, int32_t out_dtype, float* lse, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * Workspace bytes of ress_block_sparse_attn_layout: the float32 staging of
 * ress_attn_workspace_bytes (float32 inputs only), then the special rows'
 * gathered queries, outputs and lse (0 bytes when special_tokens == 0).
 * out_dtype as for the call.  0 if the shape or layout is invalid.
 */
size_t ress_attn_layout_workspace_bytes(const ress_shape* shape, const ress_layout* layout,
                                        int32_t out_dtype);

/*
 * Stage 2 with a per-view layout (VASC 4.2 and A.5).  As
 * ress_block_sparse_attn, except that
 *   - padding keys never enter a softmax;
 *   - a padding query row writes 0 and lse -inf (so does a row whose kept
 *     blocks hold no valid key);
 *   - a special query (the first special_tokens tokens of each view) attends
 *     densely to every valid key of the sequence, whatever idx says.
 *   workspace  ress_attn_layout_workspace_bytes(shape, layout, out_dtype)
 *              bytes, 256-byte aligned (NULL when that is 0).
 */
ress_status ress_block_sparse_attn_layout(const ress_shape* shape, const ress_layout* layout,
                                          const void* q, const void* k, const void* v,
                                          int32_t budget, const int32_t* idx, void* out,
                                          int32_t out_dtype, float* lse, void* workspace,
                                          size_t workspace_bytes, void* stream);

/*
 * Stage 3: drift of the dropped blocks (ReSS Abstract and Fig. 3: the drift
 * score measures how much masking a block shifts what attention writes into
 * the residual stream; the drift of a drop set depends on the directions of
 * the contributions, Fig. 9 plots quality against it).
 *
 * For query block i of head h and every dropped block j (not in idx[h][i]),
 * in ascending j order r = 0 .. nb - budget - 1:
 *   C_j[n][:] = sum_{t in block j} exp((q[n] . k[t]) / sqrt(d) - lse[h][n]) v[t][:]
 *   drift[h][i][r] = ||C_j||_F over the B x 64 matrix,
 *   set_drift[h][i] = || sum_{j dropped} C_j ||_F.
 * lse is the kept-set normaliser written by ress_block_sparse_attn for the
 * same idx.
 *
 *   idx        as for ress_block_sparse_attn, but rows must hold `budget`
 *              distinct in-range blocks (the drift row length is nb - budget).
 *              A row that names a block twice is flagged (RESS_ERR_BAD_INDEX,
 *              detail 5, via ress_check_device_errors); the drift entries
 *              such a row would place beyond nb - budget are not written.
 *   lse        [H][N] float32 from ress_block_sparse_attn.
 *   drift      out, [H][nb][nb - budget] float32 (may be NULL when budget == nb).
 *   set_drift  out, [H][nb] float32, or NULL.
 */
ress_status ress_block_drift(const ress_shape* shape, const void* q, const void* k,
                             const void* v, int32_t budget, const int32_t* idx,
                             const float* lse, float* drift, float* set_drift,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * Debug aid: checks a kept-block list on the device, ordered on `stream`
 * (VASC A.2: the binary Top-K mask has exact capacity, so a row names
 * `budget` distinct blocks; ress_select_blocks writes them ascending).
 * Launches one small kernel that reads idx and writes nothing but the device
 * error flag: RESS_ERR_BAD_INDEX, reported by ress_check_device_errors with
 * detail 80 (an entry outside [0, nb)), 81 (a row repeats a block in
 * adjacent positions) or 82 (a row not in ascending order).  The first error
 * found wins.
 *
 *   idx      [H][nb][budget] int32 device array, 4-byte aligned.
 *   budget   1 <= budget <= nb.
 */
ress_status ress_validate_idx(const ress_shape* shape, int32_t budget, const int32_t* idx,
                              void* stream);

/*
 * Stage 3 with a per-view layout (VASC 4.2 and A.5).  As ress_block_drift,
 * except that only valid keys enter a contribution and only the valid,
 * non-special queries count: the rows of padding and special queries (which
 * attend densely and drop nothing) of every C_j are zero.  lse comes from
 * ress_block_sparse_attn_layout with the same idx.
 */
ress_status ress_block_drift_layout(const ress_shape* shape, const ress_layout* layout,
                                    const void* q, const void* k, const void* v, int32_t budget,
                                    const int32_t* idx, const float* lse, float* drift,
                                    float* set_drift, void* workspace, size_t workspace_bytes,
                                    void* stream);

/*
 * Synchronises `stream`, then reports and clears the device error flag that
 * the kernels set: RESS_ERR_TIMEOUT (a device wait ran out of time),
 * RESS_ERR_BAD_INDEX (an idx entry outside [0, nb) was skipped), RESS_OK if
 * none, RESS_ERR_CUDA if the synchronisation itself failed.  `detail`, if not
 * NULL, receives a kernel-specific code of the first error (0 if none).
 */
ress_status ress_check_device_errors(void* stream, int32_t* detail);

/*
 * Name and message of the last CUDA error behind a RESS_ERR_CUDA returned to
 * the calling host thread ("" if none).  The string stays valid until the
 * thread's next library call.
 */
const char* ress_last_cuda_error(void);

/*
 * Test hook: y[i] = 2^x[i] computed by the polynomial exponential that the
 * attention kernel uses for part of its probabilities (range reduction plus
 * a degree-3 minimax polynomial on the FMA pipe; relative error <= 1e-4 for
 * -100 <= x <= 8, a finite value below 2^-99 under that).  x and y are device
 * arrays of n float32.
 */
ress_status ress_test_exp2(const float* x, float* y, int32_t n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RESS_H */

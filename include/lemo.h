/*
 * lemo.h - C ABI of liblemo.so, the sm_100a (B200) implementation of the
 * per-layer hot path of contextual token sparsity:
 *
 *   block scoring -> threshold -> compaction -> gather (selective load)
 *   -> [caller's sublayer] -> scatter with in-place residual add.
 *
 * The method is that of "Jenga: Enhancing LLM Long-Context Fine-tuning with
 * Contextual Token Sparsity" (USENIX ATC'25; called LeMo in arXiv
 * 2501.09767).  Each entry point cites the section of that paper's
 * aipaper.cc summary that defines the operation.
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 *  - bf16 tensors are passed as `uint16_t*` holding bf16 bit patterns.
 *  - "DEVICE" pointers are CUDA device (global memory) pointers on the
 *    current device; "HOST" pointers are ordinary host memory.
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  No entry point synchronises except lemo_get_error.
 *  - The caller owns and allocates every buffer, including the workspace.
 *    The library never allocates device memory.
 *  - Argument errors are detected on the host before anything is enqueued:
 *    the call returns LEMO_ERR_INVALID_ARG / LEMO_ERR_UNSUPPORTED and
 *    launches nothing.  A CUDA launch error is returned as LEMO_ERR_CUDA.
 *  - Errors that only the device can see (cu_seqlens inconsistent with the
 *    shape, an index out of range, a capacity overflow, a bounded wait that
 *    ran out) are recorded in a per-device error word and the affected work
 *    is skipped; lemo_get_error() reports and clears it.
 *  - Packed variable-length batches: sequence s occupies rows
 *    cu_seqlens[s] .. cu_seqlens[s+1]-1 of every [total_L, ...] tensor.
 *    Token blocks of `block` tokens start at each sequence's first row; the
 *    last block of a sequence may be short.  Block-indexed arrays
 *    ([total_blocks]) list all blocks of sequence 0, then sequence 1, ...,
 *    where total_blocks = sum_s ceil(L_s / block).
 */
#ifndef LEMO_H
#define LEMO_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LEMO_API __attribute__((visibility("default")))
#else
#define LEMO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lemo_status {
    LEMO_OK = 0,
    LEMO_ERR_INVALID_ARG = 1,  /* bad pointer, size, stride or cu_seqlens     */
    LEMO_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. dh = 96)    */
    LEMO_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed         */
    LEMO_ERR_CAPACITY = 4,     /* an output buffer was too small (device side) */
    LEMO_ERR_TIMEOUT = 5       /* a bounded device-side wait ran out           */
} lemo_status;

/* A cudaStream_t, passed as an opaque pointer. */
typedef void* lemo_stream;

/* Shape of one layer call on a packed batch. */
typedef struct lemo_shape {
    int32_t batch;              /* number of sequences, >= 1                       */
    const int32_t* cu_seqlens;  /* DEVICE int32 [batch+1]: 0 = cu[0] <= cu[1] <= ...
                                   <= cu[batch] = total_L (checked on device)       */
    int32_t total_L;            /* rows of the packed batch, >= 0                  */
    int32_t max_seqlen;         /* upper bound of every L_s (checked on device),
                                   0 <= max_seqlen <= 4194304                      */
    int32_t H;                  /* attention heads, >= 1                           */
    int32_t dh;                 /* head dimension: 64 or 128                       */
    int32_t block;              /* token block size b: 64 or 128                   */
} lemo_shape;

/* Human-readable name of a status code (static string). */
LEMO_API const char* lemo_status_string(lemo_status st);

/*
 * Bytes of workspace that lemo_score_blocks / lemo_select need for `shape`
 * (one buffer serves both; calls on one stream may share it).  The bound
 * covers the per-sequence plan arrays, the compaction look-back descriptors
 * and the block-score matrices when the caller passes block_max = NULL:
 * ceil(max_seqlen/b) * (total_L/b + batch) floats.  Returns 0 for an invalid
 * shape.  HOST-only computation, no CUDA call.
 */
LEMO_API size_t lemo_workspace_size(const lemo_shape* shape);

/*
 * Number of floats of the optional block_max output of lemo_score_blocks,
 * sum_s ceil(L_s/b)^2, computed from HOST sequence lengths `lengths_host`
 * [batch].  Returns 0 on a bad argument.
 */
LEMO_API int64_t lemo_block_max_elems(int32_t batch, const int32_t* lengths_host, int32_t block);

/*
 * Block-wise token informativeness scores (steps a1-a3).
 *
 * Defined by the Jenga summary, section 4.2.1: Eq. 1 (the informativeness
 * of token j sums the raw pre-softmax scores S_ij = Q_i . K_j), Eq. 2 (a
 * score block's informativeness is the maximum over its entries of the
 * per-head positive scores summed over heads and divided by N_head) and the
 * Fig. 6 caption (block scores are aggregated along the column).  Causal:
 * only pairs i > j of one sequence count (the diagonal is excluded).
 *
 *   A_ij     = (1/H) * sum_h max(scale * Q[i,h,:] . K[j,h,:], 0)
 *   M[n][m]  = max over i in block n, j in block m, j < i, of A_ij   (n >= m;
 *              0 if the block holds no such pair)
 *   score[m] = sum_{n = m}^{N_b - 1} M[n][m]                 (per sequence)
 *
 * q, k         DEVICE bf16 [total_L, H, dh] row-major (row stride H*dh),
 *              16-byte aligned.
 * scale        > 0; 1.0 gives raw Q.K (no 1/sqrt(dh)).
 * block_max    DEVICE fp32, optional (NULL = keep it in the workspace).  When
 *              given: for each sequence an [N_b, N_b] row-major matrix at
 *              offset sum_{s'<s} N_b,s'^2 (see lemo_block_max_elems); only
 *              entries with n >= m are written.
 * block_scores DEVICE fp32 [total_blocks]: score[m] of every token block.
 * ws, ws_bytes DEVICE workspace of at least lemo_workspace_size(shape) bytes,
 *              256-byte aligned, contents need no initialisation.
 *
 * The score matrix S is never written to memory: the kernel multiplies
 * Q and K tiles of one head at a time on the tensor cores (tcgen05, fp32
 * accumulation in tensor memory) and folds each head into the running
 * positive-part sum in registers; block maxima go to M, and a second pass
 * sums M's columns in a fixed order (deterministic, no float atomics).
 */
LEMO_API lemo_status lemo_score_blocks(const lemo_shape* shape, const uint16_t* q, const uint16_t* k,
                              float scale, float* block_max, float* block_scores,
                              void* ws, size_t ws_bytes, lemo_stream stream);

/*
 * Block scores of one key-tile shard of each sequence (steps a1-a3 split
 * over several GPUs for one long sequence).
 *
 * Jenga summary, section 6.4 "Scalability Analysis": the method scales over
 * GPUs without extra communication on its data path.  For a sequence too
 * long for one GPU's share of the work, the block scoring is divided by key
 * columns: the key tiles of 256 tokens of every sequence are dealt to
 * `nshards` shards in snake order (round i of nshards consecutive tiles gives
 * tile i*nshards + p to shard p when i is even, to shard nshards-1-p when i
 * is odd), so the long early columns are spread evenly.  Shard `shard`
 * computes every score tile of its key tiles - the same tiles, with the same
 * arithmetic, as lemo_score_blocks - so the column sums of its key blocks are
 * complete; it writes 0 for every other block.  The sum over all shards of
 * block_scores is therefore exactly (bit for bit) lemo_score_blocks' result:
 * one all-reduce (sum) of total_blocks floats combines the shards.
 *
 * Arguments as lemo_score_blocks, plus 0 <= shard < nshards <= 4096.
 * block_max, when given, receives only the entries of the shard's key tiles.
 * With nshards = 1 the call is lemo_score_blocks.
 */
LEMO_API lemo_status lemo_score_blocks_shard(const lemo_shape* shape, const uint16_t* q,
                                             const uint16_t* k, float scale, int32_t shard,
                                             int32_t nshards, float* block_max,
                                             float* block_scores, void* ws, size_t ws_bytes,
                                             lemo_stream stream);

/*
 * Threshold comparison and compaction of kept token ids (steps a4-a5).
 *
 * Jenga summary, section 4.2.1, "Layer-specific Threshold": the score of each
 * token block is compared with the layer's threshold and all tokens of the
 * block are retained or eliminated together.  Compaction lists the kept
 * tokens in their original order (the selective load of section 4.2.3 reads
 * them from their original positions).
 *
 *   block_mask[g] = (block_scores[g] >= threshold)       (NaN scores: 0)
 *   kept_idx      = ascending global row ids of tokens whose block is kept
 *   cu_kept[s]    = number of kept tokens in sequences 0..s-1; cu_kept[batch] = K
 *   *kept_total   = K
 *
 * block_scores DEVICE fp32 [total_blocks] (e.g. from lemo_score_blocks).
 * block_mask   DEVICE uint8 [total_blocks].
 * kept_idx     DEVICE int32 with room for total_L entries (worst case); only
 *              the first K are written.
 * cu_kept      DEVICE int32 [batch+1].   kept_total  DEVICE int32 [1].
 * ws, ws_bytes as for lemo_score_blocks.
 *
 * One pass: warp ballots and a block-wide scan count kept tokens per tile of
 * 2048 tokens, and a decoupled look-back over tile descriptors in the
 * workspace chains the tiles' offsets.  Tiles take ids from an atomic ticket,
 * so a tile only ever waits on tiles that are already running; each wait is
 * bounded in time and reports LEMO_ERR_TIMEOUT through lemo_get_error.
 * K stays on the device: nothing is copied to the host.
 */
LEMO_API lemo_status lemo_select(const lemo_shape* shape, const float* block_scores, float threshold,
                        uint8_t* block_mask, int32_t* kept_idx, int32_t* cu_kept,
                        int32_t* kept_total, void* ws, size_t ws_bytes, lemo_stream stream);

/*
 * lemo_select without a caller-provided workspace.  The paper has no
 * counterpart to this entry point; it is a deployment variant of lemo_select.
 *
 * Some callers cannot allocate device memory where they select tokens: code
 * running under a memory pool that owns the whole device and forbids further
 * cudaMalloc calls, or a latency-critical loop that must not pay for the
 * device-wide synchronisation cudaMalloc/cudaFree can imply.  This call
 * computes exactly what lemo_select computes (same arguments, outputs and
 * errors) but keeps its scratch - the per-call plan of the batch and the
 * look-back descriptors - in a 160 KB array that the library reserves in the
 * memory of every GPU it is loaded on (held until the process exits).  It
 * calls no allocating function.
 *
 * Limits: batch <= 4096 and total_L <= 16777216; a larger shape returns
 * LEMO_ERR_CAPACITY and enqueues nothing.
 * Every call looks up the array's device address on the current device (a
 * host-side query that allocates nothing).  The first call on a device may
 * also load the library's device code there; make that first call before
 * any stream capture.
 * Every call on a device uses the same array and re-initialises what must
 * start at zero at its beginning, so calls that can overlap on the GPU (for
 * example on two streams with no ordering between them) race and corrupt each
 * other's results: order them on one stream.
 */
LEMO_API lemo_status lemo_select_static_ws(const lemo_shape* shape, const float* block_scores,
                                           float threshold, uint8_t* block_mask,
                                           int32_t* kept_idx, int32_t* cu_kept,
                                           int32_t* kept_total, lemo_stream stream);

/*
 * Gather of kept rows into a zero-padded dense buffer (step a6).
 *
 * Jenga summary, section 4.2.3, "Permutation-free Token Movement" ->
 * "Selective Load": kept tokens are read straight from their original rows;
 * the zero padding of the naive path becomes a zero tail.
 *
 *   for r < K:            y[r, 0:d] = x[kept_idx[r], 0:d]   (bit copy)
 *   for K <= r < K_pad:   y[r, 0:d] = 0                     (K_pad = K rounded up to pad_to)
 *
 * x          DEVICE bf16, x_rows rows of stride ld_x elements.
 * d          row width in elements, d % 8 == 0.
 * kept_idx   DEVICE int32 [>= K], each in [0, x_rows) (checked on device).
 * kept_total DEVICE int32 [1] holding K (read on the device).
 * pad_to     >= 1.
 * y          DEVICE bf16, y_rows_capacity rows of stride ld_y; rows >= K_pad
 *            are not touched.  If K_pad > y_rows_capacity, only the first
 *            y_rows_capacity rows are written and LEMO_ERR_CAPACITY is
 *            recorded.  Size y for round_up(total_L, pad_to) rows to never
 *            need K on the host.
 * Pointers 16-byte aligned; ld_x, ld_y >= d and multiples of 8; x and y
 * must not overlap.
 */
LEMO_API lemo_status lemo_gather_pad(const uint16_t* x, int64_t ld_x, int64_t x_rows, int32_t d,
                            const int32_t* kept_idx, const int32_t* kept_total, int32_t pad_to,
                            uint16_t* y, int64_t ld_y, int64_t y_rows_capacity,
                            lemo_stream stream);

/*
 * Scatter-back fused with the residual add, in place (step a7).
 *
 * Jenga summary, section 4.2.3, "In-place Addition": the sublayer output is
 * added directly into the original input rows, which completes the padding
 * (eliminated rows are simply not touched) and the residual add in one step.
 *
 *   for r < K:  x[kept_idx[r], 0:d] = bf16_rne(float(x[kept_idx[r], :]) + float(y[r, :]))
 *   every other row of x keeps its bytes; rows of y at or beyond K are not read.
 *
 * The fp32 sum of two bf16 values rounded once to bf16 (nearest, ties to
 * even) equals the exactly rounded sum, so the result is bit-exact.
 * kept_idx entries must be distinct (lemo_select produces ascending ids) and
 * in [0, x_rows) (checked on device).  x and y must not overlap.  Alignment
 * and stride rules as for lemo_gather_pad.
 */
LEMO_API lemo_status lemo_scatter_residual(uint16_t* x, int64_t ld_x, int64_t x_rows, int32_t d,
                                  const uint16_t* y, int64_t ld_y, const int32_t* kept_idx,
                                  const int32_t* kept_total, lemo_stream stream);

/*
 * Backward-pass recomputation of the layer input (extension of step a7).
 *
 * Jenga summary, section 4.2.3, "In-place Addition": during backpropagation
 * the original inputs are recomputed by subtracting the sublayer output from
 * the output embeddings instead of being stored.
 *
 *   for r < K:  x[kept_idx[r], 0:d] = bf16_rne(float(x[kept_idx[r], :]) - float(y[r, :]))
 *   every other row of x keeps its bytes.
 *
 * One rounding of the exact difference, so the result is bit-exact; it is
 * not an exact inverse of the rounded forward addition (the recovered row is
 * within one bf16 ulp of x_out of the original).  The other passes of the
 * backward token movement reuse the forward kernels: lemo_gather_pad on the
 * output gradient gives the sublayer's output gradient at the kept rows, and
 * lemo_scatter_residual adds the sublayer's input gradient back into the
 * residual gradient.  Arguments, alignment and errors as
 * lemo_scatter_residual.
 */
LEMO_API lemo_status lemo_recompute_input(uint16_t* x, int64_t ld_x, int64_t x_rows, int32_t d,
                                          const uint16_t* y, int64_t ld_y,
                                          const int32_t* kept_idx, const int32_t* kept_total,
                                          lemo_stream stream);

/*
 * Token-block scores of the MLP block (extension of steps a1-a3).
 *
 * Jenga summary, section 4.2.1, "Extend to MLP Block": token elimination is
 * extended to the MLP using its intermediate activations - the ReLU outputs of
 * ReLU MLPs, or SiLU(gate) * up of SiLU-gated MLPs.  The page gives no
 * aggregation; the one used here is the plainest that matches Eq. 2's block
 * rule:
 *
 *   token_score[t] = sum_c max(a[t, c], 0)
 *   block_scores[g] = max over the tokens t of block g of token_score[t]
 *
 * Pass either `act` (a = act, e.g. ReLU outputs) with gate = up = NULL, or
 * `gate` and `up` with act = NULL (a = SiLU(gate) * up, SiLU(g) = g / (1 +
 * e^-g), evaluated in fp32 as g (1 + tanh(g/2)) / 2 with the hardware tanh).  All are DEVICE bf16 [total_L rows, stride ld], 16-byte
 * aligned, d_ff % 8 == 0, ld >= d_ff and ld % 8 == 0.  token_scores
 * (optional, DEVICE fp32 [total_L]) and block_scores (DEVICE fp32
 * [total_blocks]) are outputs; the block scores feed lemo_select unchanged.
 * ws as for lemo_select.  Deterministic (fixed summation order per token;
 * the block maximum does not depend on order).
 */
LEMO_API lemo_status lemo_mlp_block_scores(const lemo_shape* shape, int32_t d_ff,
                                           const uint16_t* act, const uint16_t* gate,
                                           const uint16_t* up, int64_t ld, float* token_scores,
                                           float* block_scores, void* ws, size_t ws_bytes,
                                           lemo_stream stream);

/*
 * Workspace bytes of lemo_predict_scores for `shape`, residual width d and
 * predictor rank: the plan arrays; the block means, hidden activations and
 * predicted Q/K block embeddings, each as a pair of bf16 planes hi + lo laid
 * out as tensor-core operand tiles; the split-K partial sums of the first
 * predictor GEMM; the head-group partial block products and the block-product
 * matrices; a few barrier words.  Returns 0 for invalid arguments.
 * HOST-only computation.
 */
LEMO_API size_t lemo_predict_workspace_size(const lemo_shape* shape, int32_t d, int32_t rank);

/*
 * Predicted token-block scores from low-rank ReLU predictors (step a8).
 *
 * Jenga summary, section 4.2.2, "Neural-network-based Predictor" and Eq. 3:
 * each layer has a query predictor and a key predictor that read one
 * representative embedding per token block; the product of their outputs
 * approximates the block-pair informativeness, which is aggregated along the
 * column like the exact scores.
 *
 *   xbar_g   = mean of the rows of token block g of x
 *   Qhat     = relu(xbar W1q) W2q,   Khat = relu(xbar W1k) W2k      ([blocks, H*dh])
 *   P[n][m]  = (1/H) sum_h max(Qhat_n^h . Khat_m^h, 0)   for n >= m in one sequence
 *   score[m] = sum_{n = m}^{N_b - 1} P[n][m]
 *
 * x            DEVICE bf16 [total_L rows, stride ld_x], 16-byte aligned,
 *              d % 8 == 0, ld_x >= d, ld_x % 8 == 0.
 * w1q, w1k     DEVICE bf16 [d, rank] row-major.
 * w2q, w2k     DEVICE bf16 [rank, H*dh] row-major.  Pruned predictor neurons
 *              (zero columns of W1 / rows of W2) may simply be left out by
 *              passing the compacted matrices and the smaller rank.
 * block_scores DEVICE fp32 [total_blocks].
 * ws, ws_bytes DEVICE workspace of lemo_predict_workspace_size bytes,
 *              256-byte aligned.
 * Two launches for a batch of one sequence, three otherwise: the plan
 * (written by the pooling pass itself for one sequence), a pass that streams
 * x once (bound by HBM bandwidth) and writes the block means, and one
 * persistent kernel (one CTA
 * per SM, grid-wide barriers between its phases) that runs both predictor
 * GEMMs, the Eq. 3 block products and the column sums on the tensor cores
 * (tcgen05, fp32 accumulation in tensor memory).  fp32 accuracy: every fp32
 * operand is split into bf16 hi + lo and a product is taken as hi*b + lo*b
 * (+ hi*lo' when both operands are fp32) in one fp32 accumulator; split-K and
 * head-group sums are reduced in a fixed order, so the result is
 * deterministic.  Weights need only 2-byte alignment: they are read with
 * plain loads whose width follows their alignment, with the same arithmetic.
 * A grid barrier or a tile wait that runs out reports LEMO_ERR_TIMEOUT
 * through lemo_get_error.
 */
LEMO_API lemo_status lemo_predict_scores(const lemo_shape* shape, int32_t d, const uint16_t* x,
                                         int64_t ld_x, const uint16_t* w1q, const uint16_t* w2q,
                                         const uint16_t* w1k, const uint16_t* w2k, int32_t rank,
                                         float* block_scores, void* ws, size_t ws_bytes,
                                         lemo_stream stream);

/*
 * Workspace bytes of lemo_attention_kept for `batch` sequences (the query
 * tiles of each sequence and their prefix).  Returns 0 if batch < 1.
 */
LEMO_API size_t lemo_attention_workspace_size(int32_t batch);

/*
 * Permutation-free attention over the kept tokens (extension; replaces the
 * gather -> attention -> scatter of steps a6-a7 by one kernel).
 *
 * Jenga summary, section 4.2.3, "Permutation-free Token Movement": instead
 * of eliminating, re-permuting, padding and adding back, the attention
 * kernel loads the kept tokens from their original rows (selective load) and
 * adds its output in place into the original input (in-place addition).
 * For every sequence s, kept rows r in [cu_kept[s], cu_kept[s+1]) at
 * positions kept_idx[r] (ascending) and every head h:
 *
 *   O_r^h = sum_{r' <= r, same sequence} softmax_r'(scale * Q_r^h . K_r'^h) V_r'^h
 *   x[kept_idx[r], h*dh:(h+1)*dh] = bf16(x + O_r^h)   (x != NULL: in place)
 *   o[r, h*dh:(h+1)*dh]           = bf16(O_r^h)       (o != NULL: compact)
 *
 * Exactly one of x, o is given.  Rows of x of eliminated tokens are not
 * touched; an output projection, where the model has one, is the caller's
 * (then use o, the projection GEMM and lemo_scatter_residual).
 *
 * shape        batch, cu_seqlens (DEVICE), total_L, H, dh (64 or 128),
 *              block (64 or 128) as for lemo_score_blocks.
 * q, k, v      DEVICE bf16 [total_L, H*dh], row stride ld_qkv (elements,
 *              multiple of 8), 16-byte aligned; original token order.
 * kept_idx, cu_kept, kept_total   DEVICE int32, as written by lemo_select:
 *              the kept rows must come as whole blocks of a multiple of 64
 *              tokens (a sequence's last block may be short), i.e. every 64
 *              consecutive kept rows counted from a sequence's first kept row
 *              are consecutive positions of that sequence.  A violation is
 *              reported as LEMO_ERR_INVALID_ARG by lemo_get_error.
 * scale        softmax scale (> 0), usually 1/sqrt(dh).
 * x, ld_x      DEVICE bf16 residual [total_L, >= H*dh], 16-byte aligned,
 *              must not overlap q, k or v.
 * o, ld_o      DEVICE bf16 [kept_total, >= H*dh], 16-byte aligned.
 * ws, ws_bytes DEVICE workspace of lemo_attention_workspace_size(batch)
 *              bytes, 256-byte aligned.
 * tcgen05 tensor-core kernel: fp32 scores and accumulation, probabilities
 * rounded to bf16 for the P V product, the output rounded once to bf16.
 */
LEMO_API lemo_status lemo_attention_kept(const lemo_shape* shape, const uint16_t* q,
                                         const uint16_t* k, const uint16_t* v, int64_t ld_qkv,
                                         const int32_t* kept_idx, const int32_t* cu_kept,
                                         const int32_t* kept_total, float scale, uint16_t* x,
                                         int64_t ld_x, uint16_t* o, int64_t ld_o, void* ws,
                                         size_t ws_bytes, lemo_stream stream);

/*
 * Workspace bytes of lemo_segment_loss for T tokens, vocabulary V and
 * segments of seg_rows tokens: the valid-token count, the per-token loss
 * terms, ONE segment's fp32 logits, the bf16 logit gradients of up to FOUR
 * segments (as many as there are, at most four) and the rows' partial
 * softmax statistics (8 bytes per 128 logits): about (4 + 2 x 4) x
 * min(seg_rows, T) x round_up(V, 8) bytes.  That is the activation peak that
 * segmenting divides by about T / (2 seg_rows) (it is about 6 x T x
 * round_up(V, 8) bytes unsegmented); the extra gradient segments let dW be
 * accumulated once per four segments.  Returns 0 for invalid arguments.
 * HOST-only computation.
 */
LEMO_API size_t lemo_segment_loss_workspace_size(int64_t T, int32_t V, int32_t seg_rows);

/*
 * Segment-based peak cutting of the lm-head loss (extension).
 *
 * Jenga summary, section 4.2.3, "Segment-based Peak Cutting": the final loss
 * over a large vocabulary is computed segment by segment, each segment's
 * logits are dropped as soon as its gradient is done, so the activation
 * peak falls to 1/N for N segments.  The result is that of the unsegmented
 * definition:
 *
 *   z = h W^T,  lse_t = log sum_v exp(z_tv)
 *   loss = (1/n) sum_{t valid} (lse_t - z_t,y_t),   n = #{t : y_t != ignore_index}
 *   dz_t = (softmax(z_t) - onehot(y_t)) / n   (0 for ignored tokens)
 *   dh = dz W,   dW += dz^T h
 *
 * With n = 0 the loss is 0 and the gradients are zero.
 *
 * h            DEVICE bf16 [T, d], row stride ld_h (the final hidden states).
 * w            DEVICE bf16 [V, d], row stride ld_w (the lm-head weight).
 * targets      DEVICE int32 [T]: the next-token ids, or ignore_index.
 *              A target outside [0, V) that is not ignore_index is reported
 *              as LEMO_ERR_INVALID_ARG by lemo_get_error (that token adds
 *              nothing).
 * seg_rows     tokens per segment (>= 1); the last segment may be shorter.
 * loss         DEVICE fp32 scalar (output).
 * token_loss   optional DEVICE fp32 [T]: lse_t - z_t,y_t (0 if ignored).
 * dh           optional DEVICE bf16 [T, d], row stride ld_dh (written).
 * dw           optional DEVICE fp32 [V, d], row stride ld_dw: ACCUMULATED
 *              (dW += ...), so zero it for a fresh gradient.  Pass NULL when
 *              the lm head is frozen (LoRA fine-tuning).
 * ws, ws_bytes DEVICE workspace of lemo_segment_loss_workspace_size bytes,
 *              256-byte aligned.
 * Constraints: d % 8 == 0; every stride a multiple of 8 elements and every
 * matrix 16-byte aligned; d, V, seg_rows and strides below 2^31.  With T = 0,
 * h, w and targets may be NULL (the loss is 0).
 *
 * The three GEMMs of a segment run on this library's tensor-core kernel
 * (tcgen05 on CTA pairs, bf16 inputs, fp32 accumulation in tensor memory;
 * the logits are stored in fp32, dh rounded once to bf16, dW accumulated in
 * fp32 once per four segments, in segment order); the logits GEMM's
 * epilogue also leaves each row's running (max, sum of exponentials) per
 * 128 columns, from which a separate row kernel forms the softmax, the loss
 * term and the bf16 gradient of each logit row, reading the logits once.
 * The loss is the fixed-order sum of the
 * per-token terms (deterministic); dz is rounded to bf16.
 */
LEMO_API lemo_status lemo_segment_loss(const uint16_t* h, int64_t ld_h, int64_t T, int32_t d,
                                       const uint16_t* w, int64_t ld_w, int32_t V,
                                       const int32_t* targets, int32_t ignore_index,
                                       int32_t seg_rows, float* loss, float* token_loss,
                                       uint16_t* dh, int64_t ld_dh, float* dw, int64_t ld_dw,
                                       void* ws, size_t ws_bytes, lemo_stream stream);

/*
 * Synchronises `stream`, then reports and clears the device error word of the
 * current device: LEMO_OK, LEMO_ERR_INVALID_ARG (cu_seqlens or an index
 * failed a device-side check), LEMO_ERR_CAPACITY, LEMO_ERR_TIMEOUT, or
 * LEMO_ERR_CUDA if the stream itself reported an error.
 */
LEMO_API lemo_status lemo_get_error(lemo_stream stream);

/*
 * Test hooks (process-wide, not thread-safe; for the library's own tests).
 * select_skip_publish_tile >= 0 makes that compaction tile withhold its
 * look-back descriptor so the tiles after it exhaust their bounded wait;
 * -1 disables it.  spin_limit_ns bounds every device-side wait
 * (0 restores the default of 2 s).
 */
LEMO_API void lemo_set_test_hooks(int32_t select_skip_publish_tile, int64_t spin_limit_ns);

/*
 * Test hook of lemo_predict_scores (process-wide, not thread-safe): CTA
 * `skip_cta` >= 0 of the persistent predictor kernel does not arrive at the
 * grid barrier after its first phase, so every CTA's bounded wait there runs
 * out and the call reports LEMO_ERR_TIMEOUT; -1 disables it.
 */
LEMO_API void lemo_set_predict_test_hook(int32_t skip_cta);

#ifdef __cplusplus
}
#endif

#endif /* LEMO_H */

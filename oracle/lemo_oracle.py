"""Plain float64 CPU oracle of the score -> select -> gather -> scatter path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, links or runs
this module; the CUDA library must fail loudly rather than fall back to it.
It exists so that the tests (and the benchmark's CPU-baseline leg) can check
the GPU results against a slow, obviously correct restatement of the method.

Sources (cited by page title and section / equation):

* [Jenga] "Jenga: Enhancing LLM Long-Context Fine-tuning with Contextual Token
  Sparsity", aipaper.cc summary of the USENIX ATC'25 paper.
    - §4.2.1 Eq. 1: informativeness of token j is the sum of the raw
      pre-softmax scores Q_i.K_j over the other tokens i.
    - §4.2.1 Eq. 2: a score block's informativeness is the maximum, over the
      entries of the block, of the per-head positive scores summed over heads
      and divided by N_head.
    - §4.2.1 Fig. 6 caption and "Layer-specific Threshold": block scores are
      aggregated along the column into token-block scores, which are compared
      with a layer threshold; a token block is kept or eliminated as a whole.
    - §4.2.2 Eq. 3: predicted block-pair scores are products of predicted
      query-block and key-block quantities from low-rank ReLU predictors that
      read one representative embedding per token block.
    - §4.2.3 "Permutation-free Token Movement": kept tokens are loaded from
      their original positions (selective load) and the sublayer output is
      added in place into the original input (in-place addition), which pads
      eliminated rows implicitly.
* [LeMo] pith.science reading of arXiv 2501.09767, "What carries the
  argument": the block-wise score takes the maximum positive score inside
  each block and sums across blocks by column.

Readings taken where the pages are silent or ambiguous (also listed in the
design notes of the repository):

1. Eq. 2's superscript t is the head index h.  The positive part is taken per
   head, the head sum is divided by N_head (mean over heads).
2. Causal: only pairs i > j inside one sequence count (diagonal excluded).
3. Raw Q.K with no 1/sqrt(dh); an optional positive ``scale`` multiplies S.
4. Column aggregation is a plain sum over query blocks n >= m.
5. The learned threshold of Algorithm 1 is replaced by a keep-ratio
   threshold: the midpoint between the k-th and (k+1)-th largest scores.
6. A partial last block is a short block; a block with no causal pair has
   block score 0 (every valid entry is >= 0).
7. The padded dense buffer packs all sequences' kept rows in ascending order
   with a zero tail up to a multiple of ``pad_to``.
8. The in-place residual add rounds the exact sum once to bf16 (ties to even).
9. Predictor: representative embedding = block mean of X; Eq. 3 is read per
   head with the same positive part / mean over heads as Eq. 2 and block-level
   causality n >= m (diagonal block included).
10. Backward input recomputation: x_in is recovered as bf16(x_out - y) on the
    kept rows (one rounding), which is not an exact inverse of the rounded
    forward addition.
11. MLP-block elimination: a token's informativeness is the sum of the
    positive parts of its MLP intermediate activation (the ReLU output, or
    SiLU(gate) * up); a token block's score is the maximum over its tokens,
    the block rule of Eq. 2.
12. Segment-based peak cutting: the loss is the mean next-token cross
    entropy of the lm-head logits over the tokens whose target is not the
    ignore index (0 when there is none); segmenting the tokens changes only
    the order of work, so the oracle is the unsegmented definition.
13. Permutation-free attention: the kept tokens of a sequence attend to the
    kept tokens of the same sequence at or before their own position (causal,
    self included), softmax(scale Q K^T) V per head with scale 1/sqrt(dh) by
    default; the attention output (heads concatenated, width H*dh) is added
    in place into the residual rows of the kept tokens, whose width must be
    H*dh.  An output projection, where a model has one, is the caller's.

Each function below is pinned by tests under ``tests/`` against hand-worked
values, closed forms, brute force on tiny inputs, library reductions or
invariants; none is "parity unpinned".
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "bf16_bits_to_f64",
    "f64_to_bf16_bits",
    "block_max_row",
    "score_blocks",
    "column_scores",
    "threshold_for_keep_ratio",
    "keep_mask",
    "compact",
    "gather_pad",
    "scatter_residual",
    "block_representatives",
    "predictor_embeddings",
    "predict_scores",
    "recall",
    "recompute_input",
    "mlp_token_scores",
    "mlp_block_scores",
    "lm_head_loss",
    "lm_head_loss_f64",
    "lm_head_rows",
    "attention_kept",
    "attention_residual_exact",
    "attention_kept_rows",
]

_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


# ---------------------------------------------------------------------------
# bf16 <-> float64 (the storage format of every tensor on the path)
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits) -> np.ndarray:
    """Decode bf16 bit patterns exactly into float64.

    A bf16 value is the upper 16 bits of an IEEE binary32 value, so widening
    the pattern into the top half of a 32-bit word and reading that word as
    binary32 is exact; binary32 -> float64 is exact as well.
    """
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    with np.errstate(invalid="ignore"):  # NaN patterns stay NaN
        return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x) -> np.ndarray:
    """Round float64 values to bf16 in ONE step (nearest, ties to even).

    bf16 keeps 8 significant bits; below the smallest normal (2**-126) the
    spacing is fixed at 2**-133.  The value is scaled by a power of two so
    that one unit in the last bf16 place becomes 1, rounded with ``rint``
    (ties to even) and scaled back, all exact in float64.  Magnitudes beyond
    the largest finite bf16 become infinities; NaN and infinities pass through.
    """
    x = np.asarray(x, dtype=np.float64)
    finite = np.isfinite(x)
    xf = np.where(finite, x, 0.0)
    _, e = np.frexp(xf)  # xf = m * 2**e with 0.5 <= |m| < 1
    q_exp = np.maximum(e - 8, -133)
    q = np.rint(np.ldexp(xf, -q_exp))
    val = np.ldexp(q, q_exp)
    val = np.where(np.abs(val) > _BF16_MAX, np.copysign(np.inf, val), val)
    val = np.where(finite, val, x)
    f32 = val.astype(np.float32)  # exact: every bf16 value is a binary32 value
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# a1 - a3: block-wise informativeness scores (Eq. 1, Eq. 2, Fig. 6)
# ---------------------------------------------------------------------------

def _seq_views(q_bits, k_bits, cu_seqlens, H, dh):
    q = bf16_bits_to_f64(q_bits).reshape(-1, H, dh)
    k = bf16_bits_to_f64(k_bits).reshape(-1, H, dh)
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    return q, k, cu


def block_max_row(Qs: np.ndarray, Ks: np.ndarray, n: int, block: int,
                  scale: float = 1.0) -> np.ndarray:
    """Block scores I(B^S_nm) of one query-block row n of one sequence.

    [Jenga] §4.2.1 Eq. 2 with [Jenga] Eq. 1's S_ij = Q_i.K_j:
    for every query i of block n and key j of the sequence,
    A_ij = (1/N_head) * sum_h max(scale * S^h_ij, 0); then
    I(B^S_nm) = max over the entries (i, j) of block (n, m) with j < i.

    ``Qs``/``Ks`` are float64 arrays [L, H, dh] of one sequence.  Returns a
    float64 vector of length n + 1 (key blocks m = 0..n; blocks m > n hold no
    causal pair).  A block with no causal pair (possible only for a one-token
    diagonal block) scores 0.
    """
    if not scale > 0:
        raise ValueError("scale must be positive")
    L, H, _ = Qs.shape
    r0, r1 = n * block, min((n + 1) * block, L)
    ncols = r1  # keys j < i <= r1 - 1 lie in blocks 0..n
    A = np.zeros((r1 - r0, ncols), dtype=np.float64)
    for h in range(H):
        S = scale * (Qs[r0:r1, h, :] @ Ks[:ncols, h, :].T)  # S^h_ij
        A += np.maximum(S, 0.0)  # positive part per head, summed over heads
    A /= H  # divided by N_head
    i = np.arange(r0, r1)[:, None]
    j = np.arange(ncols)[None, :]
    valid = j < i  # causal, diagonal excluded
    row = np.zeros(n + 1, dtype=np.float64)
    for m in range(n + 1):
        c0, c1 = m * block, min((m + 1) * block, ncols)
        v = valid[:, c0:c1]
        if v.any():
            row[m] = A[:, c0:c1][v].max()
    return row


def score_blocks(q_bits, k_bits, cu_seqlens, H: int, dh: int, block: int,
                 scale: float = 1.0, rows=None):
    """Per-sequence block-score matrices M[n][m] = I(B^S_nm), n >= m.

    [Jenga] §4.2.1 Eq. 2 applied to every query-block row of every sequence of
    a packed batch (tokens cu_seqlens[s] .. cu_seqlens[s+1]-1 form sequence s;
    no pair crosses a sequence boundary).  ``q_bits``/``k_bits`` are bf16 bit
    patterns [total_L, H, dh].  Returns a list of float64 [N_b, N_b] arrays
    whose strict upper triangle is 0 (those blocks hold no causal pair).

    ``rows`` (optional) restricts the work to the given (sequence, n) pairs;
    rows not listed are left as NaN.  It lets a caller evaluate a sample of a
    large problem one query-block row at a time.
    """
    q, k, cu = _seq_views(q_bits, k_bits, cu_seqlens, H, dh)
    out = []
    todo = None if rows is None else {(int(s), int(n)) for s, n in rows}
    for s in range(len(cu) - 1):
        Qs, Ks = q[cu[s]:cu[s + 1]], k[cu[s]:cu[s + 1]]
        L = cu[s + 1] - cu[s]
        nb = -(-L // block)
        M = np.zeros((nb, nb), dtype=np.float64)
        for n in range(nb):
            if todo is not None and (s, n) not in todo:
                M[n, :] = np.nan
                continue
            M[n, : n + 1] = block_max_row(Qs, Ks, n, block, scale)
        out.append(M)
    return out


def column_scores(M_list) -> np.ndarray:
    """Token-block scores I(B^T_m) = sum over query blocks n >= m of M[n][m].

    [Jenga] §4.2.1 Fig. 6 caption ("aggregated along the column") and the
    layer-specific-threshold paragraph; [LeMo] "sums across blocks by column".
    Concatenated over the sequences of the batch, in sequence order.
    """
    parts = []
    for M in M_list:
        nb = M.shape[0]
        parts.append(np.array([M[m:, m].sum() for m in range(nb)], dtype=np.float64))
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.float64)


# ---------------------------------------------------------------------------
# a4 - a5: threshold and compaction
# ---------------------------------------------------------------------------

def threshold_for_keep_ratio(scores, ratio: float) -> float:
    """Layer threshold that keeps k = floor(ratio * N + 1/2) token blocks.

    Stands in for [Jenga] Algorithm 1's learned layer thresholds (which need
    a trained model and validation accuracy): sort the layer's token-block
    scores in descending order and return the midpoint between the k-th and
    (k+1)-th largest, which keeps exactly k blocks with the widest margin.
    k = 0 gives +inf (keep none), k = N gives -inf (keep all).
    """
    s = np.sort(np.asarray(scores, dtype=np.float64))[::-1]
    N = s.size
    k = int(math.floor(ratio * N + 0.5))
    if k <= 0:
        return math.inf
    if k >= N:
        return -math.inf
    return 0.5 * (float(s[k - 1]) + float(s[k]))


def keep_mask(scores, theta) -> np.ndarray:
    """Keep bit of each token block: I(B^T_m) >= theta ([Jenga] §4.2.1, Fig. 6).

    The comparison runs in the dtype of ``scores`` (pass float32 scores and a
    float32 threshold to take the decision in the kernel's precision).
    """
    scores = np.asarray(scores)
    return (scores >= scores.dtype.type(theta)).astype(np.uint8)


def compact(mask, cu_seqlens, block: int):
    """Ascending global ids of kept tokens, per-sequence offsets and total.

    [Jenga] §4.2.1: "tokens within that block are retained or eliminated", so
    token t of sequence s lies in token block floor((t - cu[s]) / block) of
    that sequence and is kept iff that block's keep bit is set.  The kept ids
    are listed in ascending order ([Jenga] §4.2.3 selective load reads kept
    tokens from their original positions).

    Returns (kept_idx int32 [K], cu_kept int32 [B+1], K).
    """
    mask = np.asarray(mask).astype(bool)
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    kept = []
    cu_kept = [0]
    boff = 0
    for s in range(len(cu) - 1):
        L = cu[s + 1] - cu[s]
        nb = -(-L // block)
        for t in range(cu[s], cu[s + 1]):
            if mask[boff + (t - cu[s]) // block]:
                kept.append(t)
        cu_kept.append(len(kept))
        boff += nb
    if boff != mask.size:
        raise ValueError("mask length does not match the number of token blocks")
    return (np.asarray(kept, dtype=np.int32), np.asarray(cu_kept, dtype=np.int32),
            len(kept))


# ---------------------------------------------------------------------------
# a6 - a7: permutation-free token movement (§4.2.3)
# ---------------------------------------------------------------------------

def gather_pad(x_bits, kept_idx, pad_to: int) -> np.ndarray:
    """Selective load of kept rows into a zero-padded dense buffer.

    [Jenga] §4.2.3 "Selective Load": kept rows are read from their original
    positions; the naive path's zero padding becomes a zero tail.  Row r < K
    of the result is row kept_idx[r] of x, bit for bit; rows K .. K_pad-1 are
    zero, where K_pad = K rounded up to a multiple of ``pad_to``.
    """
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    K = len(kept_idx)
    K_pad = -(-K // pad_to) * pad_to
    y = np.zeros((K_pad, x_bits.shape[1]), dtype=np.uint16)
    for r in range(K):
        y[r] = x_bits[int(kept_idx[r])]
    return y


def scatter_residual(x_bits, y_bits, kept_idx) -> np.ndarray:
    """In-place residual addition of the sublayer output into x.

    [Jenga] §4.2.3 "In-place Addition": for r < K, row kept_idx[r] of x
    becomes bf16(x + y[r]) (exact sum rounded once, ties to even); every other
    row of x keeps its bytes, which is the implicit zero padding.  Returns a
    new array; the input is not modified.
    """
    x_new = np.array(x_bits, dtype=np.uint16, copy=True)
    d = x_new.shape[1]
    for r in range(len(kept_idx)):
        t = int(kept_idx[r])
        s = bf16_bits_to_f64(x_new[t]) + bf16_bits_to_f64(np.asarray(y_bits[r])[:d])
        x_new[t] = f64_to_bf16_bits(s)
    return x_new


# ---------------------------------------------------------------------------
# a8: context-aware pattern prediction (§4.2.2 Eq. 3)
# ---------------------------------------------------------------------------

def block_representatives(x_bits, cu_seqlens, block: int) -> np.ndarray:
    """Representative embedding of each token block: the mean of its rows.

    [Jenga] §4.2.2 says the predictors read "a representative embedding from
    each block" without defining it; the reading taken is the block mean of X
    (a short last block averages the rows it has).  Returns float64
    [total_blocks, d], blocks of all sequences concatenated in order.
    """
    x = bf16_bits_to_f64(x_bits)
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    reps = []
    for s in range(len(cu) - 1):
        for t0 in range(cu[s], cu[s + 1], block):
            t1 = min(t0 + block, cu[s + 1])
            reps.append(x[t0:t1].mean(axis=0))
    return np.asarray(reps, dtype=np.float64).reshape(-1, x.shape[1])


def predictor_embeddings(reps, w1_bits, w2_bits) -> np.ndarray:
    """Low-rank ReLU predictor: relu(reps @ W1) @ W2, in float64.

    [Jenga] §4.2.2 "Neural-network-based Predictor" (low-rank matrices with
    ReLU between them) with the two-matrix shape W1 [d, r], W2 [r, H*dh] of
    the workload definition.  No intermediate rounding.
    """
    w1 = bf16_bits_to_f64(w1_bits)
    w2 = bf16_bits_to_f64(w2_bits)
    return np.maximum(reps @ w1, 0.0) @ w2


def predict_scores(q_hat, k_hat, cu_seqlens, block: int, H: int, dh: int):
    """Predicted token-block scores from Eq. 3 block products.

    [Jenga] §4.2.2 Eq. 3: the block-pair score is the product of the predicted
    query-block and key-block quantities.  Read per head with Eq. 2's rules:
    P[n][m] = (1/H) * sum_h max(Qhat_n^h . Khat_m^h, 0) for n >= m (the
    diagonal block holds causal pairs, so it counts), then the column sum of
    Fig. 6.  ``q_hat``/``k_hat`` are float64 [total_blocks, H*dh].
    Returns (list of per-sequence P matrices, concatenated scores).
    """
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    qh = np.asarray(q_hat, dtype=np.float64).reshape(-1, H, dh)
    kh = np.asarray(k_hat, dtype=np.float64).reshape(-1, H, dh)
    P_list = []
    boff = 0
    for s in range(len(cu) - 1):
        nb = -(-(cu[s + 1] - cu[s]) // block)
        P = np.zeros((nb, nb), dtype=np.float64)
        for n in range(nb):
            acc = np.zeros(n + 1, dtype=np.float64)
            for h in range(H):
                acc += np.maximum(kh[boff:boff + n + 1, h, :] @ qh[boff + n, h, :], 0.0)
            P[n, : n + 1] = acc / H
        P_list.append(P)
        boff += nb
    return P_list, column_scores(P_list)


def recall(mask_pred, mask_exact) -> float:
    """|kept_pred AND kept_exact| / |kept_exact| (1.0 when nothing is kept).

    The pages report predictor recall ([Jenga] §6.2, Fig. 17(a))
    without a formula; this is the plain reading: the share of exactly-kept
    token blocks that the predicted scores also keep.
    """
    p = np.asarray(mask_pred).astype(bool)
    e = np.asarray(mask_exact).astype(bool)
    ne = int(e.sum())
    return 1.0 if ne == 0 else float((p & e).sum()) / ne


# ---------------------------------------------------------------------------
# Extensions: backward input recomputation and MLP-block elimination
# ---------------------------------------------------------------------------

def recompute_input(x_out_bits, y_bits, kept_idx) -> np.ndarray:
    """Recover the layer input from its output by subtraction.

    [Jenga] §4.2.3 "In-place Addition": during backpropagation the original
    inputs are recomputed by subtracting the sublayer output from the output
    embeddings.  For r < K, row kept_idx[r] becomes bf16(x_out - y[r]) (exact
    difference rounded once, ties to even); every other row keeps its bytes.
    """
    x_in = np.array(x_out_bits, dtype=np.uint16, copy=True)
    d = x_in.shape[1]
    for r in range(len(kept_idx)):
        t = int(kept_idx[r])
        diff = bf16_bits_to_f64(x_in[t]) - bf16_bits_to_f64(np.asarray(y_bits[r])[:d])
        x_in[t] = f64_to_bf16_bits(diff)
    return x_in


def mlp_token_scores(act_bits=None, gate_bits=None, up_bits=None) -> np.ndarray:
    """Per-token informativeness from MLP intermediate activations.

    [Jenga] §4.2.1 "Extend to MLP Block": the activations used are the ReLU
    outputs (ReLU MLPs) or SiLU(gate) * up (SiLU MLPs).  Reading taken: the
    token's score is the sum of the positive parts of that vector.  Pass
    either ``act_bits`` (bf16 [L, d_ff], used as is) or ``gate_bits`` and
    ``up_bits`` (bf16 [L, d_ff]; SiLU(g) = g / (1 + exp(-g)) in float64).
    """
    if act_bits is not None:
        a = bf16_bits_to_f64(act_bits)
    else:
        g = bf16_bits_to_f64(gate_bits)
        u = bf16_bits_to_f64(up_bits)
        a = g / (1.0 + np.exp(-g)) * u
    return np.maximum(a, 0.0).sum(axis=1)


def mlp_block_scores(token_scores, cu_seqlens, block: int) -> np.ndarray:
    """Token-block score of the MLP path: the maximum over the block's tokens
    (Eq. 2's block rule), blocks of all sequences concatenated in order."""
    ts = np.asarray(token_scores, dtype=np.float64)
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    out = []
    for s in range(len(cu) - 1):
        for t0 in range(cu[s], cu[s + 1], block):
            out.append(ts[t0:min(t0 + block, cu[s + 1])].max())
    return np.asarray(out, dtype=np.float64)


# ---------------------------------------------------------------------------
# Extension: segment-based peak cutting of the lm-head loss (§4.2.3)
# ---------------------------------------------------------------------------

def lm_head_loss(h_bits, w_bits, targets, ignore_index: int = -100):
    """Mean cross entropy of the lm-head logits and its gradients, float64.

    [Jenga] §4.2.3 "Segment-based Peak Cutting": each token's logits over the
    vocabulary feed a next-token loss; the pages split the tokens into
    segments and finish each segment's gradient before the next one, which
    changes the peak memory but not the result.  This is the plain
    definition the segmented computation must reproduce:

        z        = h W^T                        (logits, [T, V])
        lse_t    = log sum_v exp(z_tv)
        loss     = (1/n) sum_{t valid} (lse_t - z_t,y_t),  n = #valid tokens
        dz_t     = (softmax(z_t) - onehot(y_t)) / n   (0 for ignored tokens)
        dh       = dz W,   dW = dz^T h

    ``h_bits`` bf16 [T, d], ``w_bits`` bf16 [V, d] (the lm-head weight),
    ``targets`` int [T]; a target equal to ``ignore_index`` is ignored.  With
    no valid token the loss and both gradients are 0.
    Returns (loss, dh [T, d], dW [V, d], lse [T]) in float64.
    """
    return lm_head_loss_f64(bf16_bits_to_f64(h_bits), bf16_bits_to_f64(w_bits), targets,
                            ignore_index)


def lm_head_loss_f64(h, w, targets, ignore_index: int = -100):
    """``lm_head_loss`` on float64 arrays h [T, d], w [V, d] (no bf16 decode)."""
    h = np.asarray(h, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    y = np.asarray(targets, dtype=np.int64)
    T, V = h.shape[0], w.shape[0]
    valid = y != ignore_index
    if np.any((y[valid] < 0) | (y[valid] >= V)):
        raise ValueError("target outside [0, V)")
    z = h @ w.T
    zmax = z.max(axis=1, keepdims=True)
    lse = (zmax + np.log(np.exp(z - zmax).sum(axis=1, keepdims=True)))[:, 0]
    n = int(valid.sum())
    if n == 0:
        return 0.0, np.zeros_like(h), np.zeros_like(w), lse
    rows = np.nonzero(valid)[0]
    loss = float((lse[rows] - z[rows, y[rows]]).sum() / n)
    dz = np.exp(z - lse[:, None])
    dz[rows, y[rows]] -= 1.0
    dz[~valid] = 0.0
    dz /= n
    return loss, dz @ w, dz.T @ h, lse


def lm_head_rows(h_bits, w_bits, targets, rows, n_valid: int, ignore_index: int = -100):
    """Per-token terms of ``lm_head_loss`` for the listed token rows only.

    For each t in ``rows``: (lse_t - z_t,y_t) (0 if ignored) and the row dh_t
    = dz_t W, with dz_t scaled by 1/``n_valid`` (the valid-token count of the
    whole batch).  The same definition as ``lm_head_loss``, evaluated one row
    at a time so that sampled rows of a large workload stay cheap.
    Returns (per-row loss terms [len(rows)], dh rows [len(rows), d]).
    """
    w = bf16_bits_to_f64(w_bits)
    out_l, out_dh = [], []
    for t in rows:
        ht = bf16_bits_to_f64(np.asarray(h_bits)[int(t)])
        z = w @ ht
        m = z.max()
        lse = m + math.log(np.exp(z - m).sum())
        yt = int(targets[int(t)])
        if yt == ignore_index or n_valid == 0:
            out_l.append(0.0)
            out_dh.append(np.zeros(w.shape[1]))
            continue
        p = np.exp(z - lse)
        p[yt] -= 1.0
        out_l.append(lse - z[yt])
        out_dh.append((p / n_valid) @ w)
    return np.asarray(out_l), np.asarray(out_dh).reshape(len(out_l), w.shape[1])


# ---------------------------------------------------------------------------
# Extension: permutation-free attention over the kept tokens (§4.2.3)
# ---------------------------------------------------------------------------

def attention_kept(q_bits, k_bits, v_bits, kept_idx, cu_kept, H: int, dh: int,
                   scale: float | None = None) -> np.ndarray:
    """Causal multi-head attention among the kept tokens, float64.

    [Jenga] §4.2.3 "Permutation-free Token Movement": the attention reads the
    kept tokens directly from their original rows (selective load) instead
    of a re-permuted copy.  Kept rows r of sequence s are
    kept_idx[cu_kept[s] : cu_kept[s+1]] (ascending positions); query r
    attends to the kept keys r' of the same sequence with position
    kept_idx[r'] <= kept_idx[r]:

        O_r^h = sum_{r'} softmax_r'(scale * Q_r^h . K_r'^h) V_r'^h

    ``q_bits``, ``k_bits``, ``v_bits``: bf16 [total_L, H*dh] in original token
    order; scale defaults to 1/sqrt(dh).  Returns float64 [K, H*dh], row r
    the output of kept token r.
    """
    if scale is None:
        scale = 1.0 / math.sqrt(dh)
    idx = np.asarray(kept_idx, dtype=np.int64)
    cu = [int(c) for c in np.asarray(cu_kept)]
    K = len(idx)
    out = np.zeros((K, H * dh), dtype=np.float64)
    for s in range(len(cu) - 1):
        rows = idx[cu[s]:cu[s + 1]]
        if len(rows) == 0:
            continue
        q = bf16_bits_to_f64(np.asarray(q_bits)[rows]).reshape(-1, H, dh)
        k = bf16_bits_to_f64(np.asarray(k_bits)[rows]).reshape(-1, H, dh)
        v = bf16_bits_to_f64(np.asarray(v_bits)[rows]).reshape(-1, H, dh)
        n = len(rows)
        allowed = rows[None, :] <= rows[:, None]  # key position <= query position
        for h in range(H):
            logits = scale * (q[:, h, :] @ k[:, h, :].T)
            logits = np.where(allowed, logits, -np.inf)
            m = logits.max(axis=1, keepdims=True)
            p = np.exp(logits - m)
            p /= p.sum(axis=1, keepdims=True)
            out[cu[s]:cu[s] + n, h * dh:(h + 1) * dh] = p @ v[:, h, :]
    return out


def attention_residual_exact(x_bits, o, kept_idx) -> np.ndarray:
    """The in-place addition of the attention output before rounding.

    [Jenga] §4.2.3 "In-place Addition": row kept_idx[r] of x receives
    x + O_r; every other row keeps its value.  Returns float64 [rows, d] (the
    exact sums; the stored result is their bf16 rounding).
    """
    x = bf16_bits_to_f64(x_bits).copy()
    idx = np.asarray(kept_idx, dtype=np.int64)
    x[idx] += np.asarray(o, dtype=np.float64)
    return x


def attention_kept_rows(q_bits, k_bits, v_bits, kept_idx, cu_kept, H: int, dh: int, rows,
                        scale: float | None = None) -> np.ndarray:
    """``attention_kept`` evaluated for the listed compact rows only (the same
    definition, one query row at a time, for sampled rows of large inputs).
    Returns float64 [len(rows), H*dh]."""
    if scale is None:
        scale = 1.0 / math.sqrt(dh)
    idx = np.asarray(kept_idx, dtype=np.int64)
    cu = np.asarray(cu_kept, dtype=np.int64)
    out = np.zeros((len(rows), H * dh), dtype=np.float64)
    for n, r in enumerate(rows):
        s = int(np.searchsorted(cu, r, side="right")) - 1
        keys = idx[cu[s]:r + 1]  # kept keys of the sequence up to row r (ascending)
        q = bf16_bits_to_f64(np.asarray(q_bits)[idx[r]]).reshape(H, dh)
        k = bf16_bits_to_f64(np.asarray(k_bits)[keys]).reshape(-1, H, dh)
        v = bf16_bits_to_f64(np.asarray(v_bits)[keys]).reshape(-1, H, dh)
        for h in range(H):
            logits = scale * (k[:, h, :] @ q[h])
            p = np.exp(logits - logits.max())
            out[n, h * dh:(h + 1) * dh] = (p / p.sum()) @ v[:, h, :]
    return out

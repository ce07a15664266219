"""Pins for the CPU oracle: each check ties it to something other than itself.

* hand-worked values of Eq. 2 (tests/golden/hand_examples.json),
* brute-force per-entry loops in pure Python on tiny integer inputs,
* closed forms (all-ones inputs), a library reduction (block size 1),
* invariants (positive homogeneity, head permutation, popcount, scatter of a
  gather, untouched rows, zero tail),
* an exhaustive check of the bf16 codec and an independent rounding route.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
from contextual_token_sparsity_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(a):
    """Exact bf16 bits of small values (integers / halves) via float32."""
    return synth.to_bf16_bits(np.asarray(a, dtype=np.float32))


# ---------------------------------------------------------------- bf16 codec

def test_bf16_roundtrip_all_patterns():
    allb = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = oracle.bf16_bits_to_f64(allb)
    back = oracle.f64_to_bf16_bits(v)
    finite = np.isfinite(v)
    assert np.array_equal(back[finite], allb[finite])
    inf = np.isinf(v)
    assert np.array_equal(back[inf], allb[inf])
    assert np.isnan(oracle.bf16_bits_to_f64(back[np.isnan(v)])).all()


def test_bf16_rounding_against_brute_neighbours():
    """Nearest bf16 (ties to even) by searching the sorted table of all finite
    bf16 values: independent of the frexp/rint route inside the oracle."""
    allb = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = oracle.bf16_bits_to_f64(allb)
    fin = np.isfinite(vals) & ~((vals == 0) & (np.signbit(vals)))  # drop -0
    table_v = vals[fin]
    table_b = allb[fin]
    order = np.argsort(table_v, kind="stable")
    table_v, table_b = table_v[order], table_b[order]
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        # exact midpoints between neighbours (ties)
        0.5 * (table_v[1000:1400] + table_v[1001:1401]),
        0.5 * (table_v[-600:-200] + table_v[-599:-199]),
        rng.standard_normal(2000) * 1e-39,  # subnormal range
    ])
    got = oracle.f64_to_bf16_bits(x)
    pos = np.searchsorted(table_v, x)
    for xi, gi, p in zip(x, got, pos):
        lo = table_v[max(p - 1, 0)]
        hi = table_v[min(p, table_v.size - 1)]
        dlo, dhi = abs(xi - lo), abs(hi - xi)
        if dlo < dhi:
            want = table_b[max(p - 1, 0)]
        elif dhi < dlo:
            want = table_b[min(p, table_v.size - 1)]
        else:  # tie: even mantissa (lowest bit of the pattern is 0)
            a, b = table_b[max(p - 1, 0)], table_b[min(p, table_v.size - 1)]
            want = a if (int(a) & 1) == 0 else b
        if want == 0 and xi < 0:
            want = 0x8000  # -0 keeps its sign
        assert int(gi) == int(want), (xi, hex(gi), hex(want))


def test_bf16_overflow_and_specials():
    mx = (2 - 2 ** -7) * 2.0 ** 127
    half_ulp = 2.0 ** 119
    got = oracle.f64_to_bf16_bits([mx, mx + half_ulp * 0.99, mx + half_ulp, -(mx + half_ulp),
                                   np.inf, -np.inf, 0.0, -0.0])
    assert [hex(int(g)) for g in got] == ["0x7f7f", "0x7f7f", "0x7f80", "0xff80",
                                         "0x7f80", "0xff80", "0x0", "0x8000"]


# ------------------------------------------------------------- hand examples

def _hand_cases():
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _hand_cases(), ids=lambda c: c["name"])
def test_hand_worked_examples(case):
    H, dh, b = case["H"], case["dh"], case["block"]
    q = bits(case["q"]).reshape(-1, H * dh)
    k = bits(case["k"]).reshape(-1, H * dh)
    cu = np.array([0, q.shape[0]], dtype=np.int32)
    M = oracle.score_blocks(q, k, cu, H, dh, b)
    np.testing.assert_array_equal(M[0], np.array(case["M"]))
    sc = oracle.column_scores(M)
    np.testing.assert_array_equal(sc, np.array(case["scores"]))
    if "scores_if_diagonal_included" in case:
        assert not np.array_equal(sc, case["scores_if_diagonal_included"])
        assert not np.array_equal(sc, case["scores_if_non_causal"])


# ---------------------------------------------------------------- brute force

def brute_scores(qf, kf, cu, H, dh, b):
    """Per-entry loops in pure Python: Eq. 1 / Eq. 2 / Fig. 6 with i > j."""
    Ms, scores = [], []
    for s in range(len(cu) - 1):
        o, L = cu[s], cu[s + 1] - cu[s]
        nb = -(-L // b)
        M = [[0.0] * nb for _ in range(nb)]
        for i in range(L):
            for j in range(i):
                a = 0.0
                for h in range(H):
                    sv = 0.0
                    for t in range(dh):
                        sv += qf[o + i][h][t] * kf[o + j][h][t]
                    if sv > 0:
                        a += sv
                a = a / H
                n, m = i // b, j // b
                if a > M[n][m]:
                    M[n][m] = a
        Ms.append(M)
        for m in range(nb):
            scores.append(sum(M[n][m] for n in range(m, nb)))
    return Ms, scores


@pytest.mark.parametrize("seed,lengths,H,dh,b", [
    (0, [16], 1, 1, 1),
    (1, [13], 2, 3, 2),
    (2, [16], 3, 4, 4),
    (3, [5, 0, 11, 1, 7], 2, 2, 4),
    (4, [9, 16], 4, 4, 2),
    (5, [3], 1, 2, 4),
])
def test_scores_match_brute_force(seed, lengths, H, dh, b):
    rng = np.random.default_rng(seed)
    total = sum(lengths)
    qi = rng.integers(-3, 4, size=(total, H, dh))
    ki = rng.integers(-3, 4, size=(total, H, dh))
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    Ms, want = brute_scores(qi.tolist(), ki.tolist(), cu.tolist(), H, dh, b)
    got_M = oracle.score_blocks(bits(qi).reshape(total, -1), bits(ki).reshape(total, -1),
                                cu, H, dh, b)
    for gm, bm in zip(got_M, Ms):
        np.testing.assert_allclose(gm, np.array(bm).reshape(gm.shape), rtol=1e-13, atol=0)
    got = oracle.column_scores(got_M)
    np.testing.assert_allclose(got, np.array(want), rtol=1e-13, atol=0)


# ------------------------------------------------------ closed forms, library

@pytest.mark.parametrize("L,H,dh,b", [(256, 2, 8, 64), (200, 3, 16, 64), (130, 1, 4, 128), (129, 2, 4, 64)])
def test_all_ones_closed_form(L, H, dh, b):
    q = bits(np.ones((L, H * dh)))
    cu = np.array([0, L], dtype=np.int32)
    M = oracle.score_blocks(q, q, cu, H, dh, b)[0]
    nb = -(-L // b)
    last_len = L - (nb - 1) * b
    for n in range(nb):
        for m in range(n + 1):
            empty = (n == m and (b if n < nb - 1 else last_len) < 2)
            assert M[n, m] == (0.0 if empty else float(dh))
    sc = oracle.column_scores([M])
    want = [(nb - m) * dh - (dh if (m == nb - 1 and last_len < 2) else 0) for m in range(nb)]
    np.testing.assert_array_equal(sc, np.array(want, dtype=np.float64))


@pytest.mark.parametrize("seed", [0, 1])
def test_block_size_one_reduces_to_matmul(seed):
    """b = 1, H = 1: score_j = sum_{i > j} relu((Q K^T)_ij), a library product."""
    rng = np.random.default_rng(seed)
    L, dh = 40, 8
    qb = synth.to_bf16_bits(rng.standard_normal((L, dh)))
    kb = synth.to_bf16_bits(rng.standard_normal((L, dh)))
    Q, K = synth.bf16_bits_to_f32(qb).astype(np.float64), synth.bf16_bits_to_f32(kb).astype(np.float64)
    want = np.tril(np.maximum(Q @ K.T, 0.0), -1).sum(axis=0)
    got = oracle.column_scores(oracle.score_blocks(qb, kb, np.array([0, L]), 1, dh, 1))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_positive_values_reduce_to_eq1():
    """All-positive Q, K, b = 1, H = 1: the score is Eq. 1 restricted to i > j."""
    rng = np.random.default_rng(3)
    L, dh = 24, 4
    qb = bits(rng.integers(1, 5, size=(L, dh)))
    kb = bits(rng.integers(1, 5, size=(L, dh)))
    Q = synth.bf16_bits_to_f32(qb).astype(np.float64)
    K = synth.bf16_bits_to_f32(kb).astype(np.float64)
    S = Q @ K.T
    want = [sum(S[i, j] for i in range(L) if i > j) for j in range(L)]
    got = oracle.column_scores(oracle.score_blocks(qb, kb, np.array([0, L]), 1, dh, 1))
    np.testing.assert_array_equal(got, np.array(want))


# ----------------------------------------------------------------- invariants

def _rand_qk(seed, L, H, dh):
    rng = np.random.default_rng(seed)
    return (synth.to_bf16_bits(rng.standard_normal((L, H * dh))),
            synth.to_bf16_bits(rng.standard_normal((L, H * dh))))


def test_positive_homogeneity_and_scale():
    q, k = _rand_qk(11, 150, 3, 8)
    cu = np.array([0, 150])
    base = oracle.column_scores(oracle.score_blocks(q, k, cu, 3, 8, 64))
    q4 = oracle.f64_to_bf16_bits(4.0 * oracle.bf16_bits_to_f64(q))  # exact: power of two
    s4 = oracle.column_scores(oracle.score_blocks(q4, k, cu, 3, 8, 64))
    np.testing.assert_allclose(s4, 4.0 * base, rtol=1e-13)
    sc = oracle.column_scores(oracle.score_blocks(q, k, cu, 3, 8, 64, scale=0.125))
    np.testing.assert_allclose(sc, 0.125 * base, rtol=1e-13)
    assert (base >= 0).all()
    with pytest.raises(ValueError):
        oracle.score_blocks(q, k, cu, 3, 8, 64, scale=-1.0)


def test_head_permutation_invariance():
    H, dh, L = 4, 8, 130
    q, k = _rand_qk(12, L, H, dh)
    perm = [2, 0, 3, 1]
    qp = q.reshape(L, H, dh)[:, perm].reshape(L, -1)
    kp = k.reshape(L, H, dh)[:, perm].reshape(L, -1)
    cu = np.array([0, L])
    a = oracle.column_scores(oracle.score_blocks(q, k, cu, H, dh, 64))
    b = oracle.column_scores(oracle.score_blocks(qp, kp, cu, H, dh, 64))
    np.testing.assert_allclose(a, b, rtol=1e-13)


def test_zero_queries_give_zero_scores():
    q, k = _rand_qk(13, 100, 2, 8)
    z = np.zeros_like(q)
    sc = oracle.column_scores(oracle.score_blocks(z, k, np.array([0, 100]), 2, 8, 64))
    assert (sc == 0).all()


def test_sequences_do_not_interact():
    q, k = _rand_qk(14, 300, 2, 8)
    cu = np.array([0, 100, 300])
    packed = oracle.column_scores(oracle.score_blocks(q, k, cu, 2, 8, 64))
    a = oracle.column_scores(oracle.score_blocks(q[:100], k[:100], np.array([0, 100]), 2, 8, 64))
    b = oracle.column_scores(oracle.score_blocks(q[100:], k[100:], np.array([0, 200]), 2, 8, 64))
    np.testing.assert_array_equal(packed, np.concatenate([a, b]))


def test_rows_sample_matches_full():
    q, k = _rand_qk(15, 400, 2, 8)
    cu = np.array([0, 250, 400])
    full = oracle.score_blocks(q, k, cu, 2, 8, 64)
    part = oracle.score_blocks(q, k, cu, 2, 8, 64, rows=[(0, 3), (1, 1)])
    np.testing.assert_array_equal(part[0][3], full[0][3])
    np.testing.assert_array_equal(part[1][1], full[1][1])
    assert np.isnan(part[0][0]).all()


# ------------------------------------------------------ threshold + compaction

def test_threshold_keeps_exactly_k():
    rng = np.random.default_rng(5)
    s = rng.random(256)
    for r, k in [(0.3, 77), (0.5, 128), (0.7, 179), (0.0, 0), (1.0, 256)]:
        th = oracle.threshold_for_keep_ratio(s, r)
        assert int(oracle.keep_mask(s, th).sum()) == k


def test_threshold_half_is_linear_median():
    s = np.random.default_rng(6).random(16)
    assert math.isclose(oracle.threshold_for_keep_ratio(s, 0.5), float(np.percentile(s, 50)),
                        rel_tol=0, abs_tol=1e-15)


def test_keep_mask_ties_keep():
    assert list(oracle.keep_mask(np.array([1.0, 2.0, 2.0, 3.0]), 2.0)) == [0, 1, 1, 1]


@pytest.mark.parametrize("lengths,b", [([256], 64), ([100, 0, 37, 64], 64), ([300, 129], 128)])
def test_compact_invariants(lengths, b):
    rng = np.random.default_rng(len(lengths))
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    nbs = [-(-L // b) for L in lengths]
    mask = rng.integers(0, 2, size=sum(nbs)).astype(np.uint8)
    idx, cu_kept, K = oracle.compact(mask, cu, b)
    assert K == len(idx) == cu_kept[-1]
    assert (np.diff(idx) > 0).all()
    # kept count = sum of the kept blocks' lengths (b * popcount for full blocks)
    want_K, off = 0, 0
    for s, L in enumerate(lengths):
        for m in range(nbs[s]):
            if mask[off + m]:
                want_K += min(b, L - m * b)
        off += nbs[s]
        assert cu_kept[s + 1] - cu_kept[s] == sum(1 for t in idx if cu[s] <= t < cu[s + 1])
    assert K == want_K
    # membership by brute force
    kept = set(int(t) for t in idx)
    off = 0
    for s, L in enumerate(lengths):
        for t in range(L):
            assert (cu[s] + t in kept) == bool(mask[off + t // b])
        off += nbs[s]


def test_compact_full_blocks_popcount():
    mask = np.array([1, 0, 1, 1, 0, 0, 1, 0], dtype=np.uint8)
    idx, cu_kept, K = oracle.compact(mask, np.array([0, 512]), 64)
    assert K == 64 * int(mask.sum())


# -------------------------------------------------------- gather / scatter

def test_gather_then_scatter_doubles_kept_rows():
    rng = np.random.default_rng(21)
    x = synth.to_bf16_bits(rng.standard_normal((300, 24)))
    mask = np.array([1, 0, 1, 1, 0], dtype=np.uint8)
    idx, _, K = oracle.compact(mask, np.array([0, 300]), 64)
    y = oracle.gather_pad(x, idx, 128)
    assert y.shape[0] == -(-K // 128) * 128
    assert (y[K:] == 0).all()  # zero tail rows are 0x0000
    xn = oracle.scatter_residual(x, y, idx)
    kept = np.zeros(300, bool)
    kept[idx] = True
    assert np.array_equal(xn[~kept], x[~kept])  # eliminated rows untouched
    two_x = synth.to_bf16_bits(2.0 * synth.bf16_bits_to_f32(x[kept]))  # exact doubling
    assert np.array_equal(xn[kept], two_x)


def test_scatter_single_rounding_equals_f32_route():
    """bf16(x + y) from the exact sum equals float32 add then one RNE to bf16
    (the route a GPU takes), including wide exponent gaps and ties."""
    rng = np.random.default_rng(22)
    n = 200000
    a = synth.to_bf16_bits(rng.standard_normal(n) * 2.0 ** rng.integers(-40, 40, n))
    b = synth.to_bf16_bits(rng.standard_normal(n) * 2.0 ** rng.integers(-40, 40, n))
    want = oracle.scatter_residual(a.reshape(-1, 1), b.reshape(-1, 1), np.arange(n))[:, 0]
    f32 = synth.bf16_bits_to_f32(a) + synth.bf16_bits_to_f32(b)
    got = synth.to_bf16_bits(f32)
    assert np.array_equal(got, want)


# ------------------------------------------------------------------- predictor

def test_block_representatives_brute():
    rng = np.random.default_rng(30)
    x = synth.to_bf16_bits(rng.standard_normal((10, 3)))
    reps = oracle.block_representatives(x, np.array([0, 7, 10]), 4)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    want = [xf[0:4].mean(0), xf[4:7].mean(0), xf[7:10].mean(0)]
    np.testing.assert_allclose(reps, np.array(want), rtol=1e-15)


def test_predictor_identity_weights_match_exact_scores_on_block_means():
    """W1 = [I, -I], W2 = [I; -I] make the predictor output the block mean
    itself, so Eq. 3's products below the diagonal equal Eq. 2 on the
    sequence of block means with block size 1; the diagonal block is
    (1/H) sum_h ||xbar_n^h||^2."""
    rng = np.random.default_rng(31)
    H, dh, b, L = 2, 4, 4, 24
    d = H * dh
    x = synth.to_bf16_bits(rng.integers(-4, 5, size=(L, d)).astype(np.float64))
    eye = np.eye(d)
    w1 = synth.to_bf16_bits(np.concatenate([eye, -eye], axis=1))
    w2 = synth.to_bf16_bits(np.concatenate([eye, -eye], axis=0))
    cu = np.array([0, L])
    reps = oracle.block_representatives(x, cu, b)
    emb = oracle.predictor_embeddings(reps, w1, w2)
    np.testing.assert_allclose(emb, reps, rtol=0, atol=1e-15)
    P, sc = oracle.predict_scores(emb, emb, cu, b, H, dh)
    nb = L // b
    # block means are multiples of 1/4 -> exact in bf16
    rb = synth.to_bf16_bits(reps)
    M = oracle.score_blocks(rb, rb, np.array([0, nb]), H, dh, 1)[0]
    for n in range(nb):
        for m in range(n):
            assert P[0][n, m] == pytest.approx(M[n, m], rel=1e-14, abs=1e-14)
        diag = np.mean([np.dot(reps[n, h * dh:(h + 1) * dh], reps[n, h * dh:(h + 1) * dh])
                        for h in range(H)])
        assert P[0][n, n] == pytest.approx(diag, rel=1e-14)


def test_predictor_zeroed_neurons_drop_out():
    d, r, out = 64, 32, 16
    w1, w2, live = synth.predictor_weights(d, r, out, 0.4, seed=1, stream=10)
    assert len(live) == r - int(0.4 * r)
    reps = np.random.default_rng(2).standard_normal((9, d))
    full = oracle.predictor_embeddings(reps, w1, w2)
    compact_ = oracle.predictor_embeddings(reps, w1[:, live], w2[live, :])
    np.testing.assert_allclose(full, compact_, rtol=1e-13, atol=1e-13)


def test_predict_scores_brute():
    rng = np.random.default_rng(33)
    H, dh = 2, 3
    qh = rng.standard_normal((5, H * dh))
    kh = rng.standard_normal((5, H * dh))
    cu = np.array([0, 10, 15])  # blocks of 4: 3 + 2 blocks
    P, sc = oracle.predict_scores(qh, kh, cu, 4, H, dh)
    want = []
    for (b0, nb) in [(0, 3), (3, 2)]:
        for m in range(nb):
            tot = 0.0
            for n in range(m, nb):
                a = 0.0
                for h in range(H):
                    v = sum(qh[b0 + n, h * dh + t] * kh[b0 + m, h * dh + t] for t in range(dh))
                    a += max(v, 0.0)
                tot += a / H
            want.append(tot)
    np.testing.assert_allclose(sc, want, rtol=1e-13)


def test_recall():
    assert oracle.recall([1, 0, 1, 1], [1, 1, 0, 1]) == pytest.approx(2 / 3)
    assert oracle.recall([0, 0], [0, 0]) == 1.0


# --------------------------------------------- backward recompute, MLP scores

def test_recompute_input_inverts_exact_additions():
    """Small integers: x_out = x_in + y is exact, so subtraction recovers x_in."""
    rng = np.random.default_rng(40)
    x_in = bits(rng.integers(-50, 50, size=(200, 16)))
    idx = np.arange(0, 200, 3, dtype=np.int32)
    y = bits(rng.integers(-50, 50, size=(len(idx), 16)))
    x_out = oracle.scatter_residual(x_in, y, idx)
    assert np.array_equal(oracle.recompute_input(x_out, y, idx), x_in)


def test_recompute_input_error_bound_and_untouched_rows():
    """In general the recovered row is within one bf16 ulp of x_out of the
    original (one rounding in each direction), and other rows keep their bytes."""
    rng = np.random.default_rng(41)
    x_in = synth.to_bf16_bits(rng.standard_normal((300, 32)))
    idx = np.arange(1, 300, 2, dtype=np.int32)
    y = synth.to_bf16_bits(rng.standard_normal((len(idx), 32)) * 10 ** rng.uniform(-2, 2, (len(idx), 1)))
    x_out = oracle.scatter_residual(x_in, y, idx)
    rec = oracle.recompute_input(x_out, y, idx)
    keep = np.ones(300, bool)
    keep[idx] = False
    assert np.array_equal(rec[keep], x_out[keep])
    xo = oracle.bf16_bits_to_f64(x_out[idx])
    ulp = np.ldexp(1.0, np.frexp(np.abs(xo) + 1e-300)[1] - 8)
    err = np.abs(oracle.bf16_bits_to_f64(rec[idx]) - oracle.bf16_bits_to_f64(x_in[idx]))
    assert (err <= ulp + 1e-300).all()
    # and the definition: one rounding of the exact difference, via float32
    f32 = synth.bf16_bits_to_f32(x_out[idx]) - synth.bf16_bits_to_f32(y)
    assert np.array_equal(rec[idx], synth.to_bf16_bits(f32))


def test_mlp_scores_brute_force():
    rng = np.random.default_rng(42)
    a = bits(rng.integers(-4, 5, size=(10, 6)))
    af = synth.bf16_bits_to_f32(a).astype(np.float64)
    want = [sum(max(v, 0.0) for v in row) for row in af]
    np.testing.assert_array_equal(oracle.mlp_token_scores(act_bits=a), want)
    cu = np.array([0, 7, 10])
    blocks = oracle.mlp_block_scores(want, cu, 4)
    np.testing.assert_array_equal(blocks, [max(want[0:4]), max(want[4:7]), max(want[7:10])])


def test_mlp_silu_gate_matches_relu_path_and_closed_form():
    rng = np.random.default_rng(43)
    g = synth.to_bf16_bits(rng.standard_normal((5, 8)) * 3)
    u = synth.to_bf16_bits(rng.standard_normal((5, 8)))
    gf = synth.bf16_bits_to_f32(g).astype(np.float64)
    uf = synth.bf16_bits_to_f32(u).astype(np.float64)
    silu = gf * (0.5 * (1.0 + np.tanh(0.5 * gf)))  # logistic via tanh: an independent route
    want = np.maximum(silu * uf, 0.0).sum(axis=1)
    np.testing.assert_allclose(oracle.mlp_token_scores(gate_bits=g, up_bits=u), want, rtol=1e-13)
    # gate = 0: SiLU(0) = 0, every score is 0
    z = np.zeros_like(g)
    assert (oracle.mlp_token_scores(gate_bits=z, up_bits=u) == 0).all()

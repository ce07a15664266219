"""Pins of the oracle's attention over kept tokens (permutation-free movement).

Checked against: torch's fp64 scaled-dot-product attention on the gathered
rows (a library routine of the same definition), a pure-Python per-row
softmax on tiny inputs, closed forms (constant V, zero Q gives running means
of V over the kept keys), and invariants (keeping every token is plain causal
attention; sequences do not see each other; eliminated rows of x stay).
"""

import math

import numpy as np
import pytest

import oracle
from contextual_token_sparsity_b200 import synth


def _qkv(L, H, dh, seed, scale=1.0):
    r = np.random.default_rng(seed)
    f = lambda: synth.to_bf16_bits(r.standard_normal((L, H * dh)) * scale)  # noqa: E731
    return f(), f(), f()


def _kept(lengths, b, seed):
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    nb = sum(-(-L // b) for L in lengths)
    mask = np.random.default_rng(seed).integers(0, 2, nb).astype(np.uint8)
    idx, cu_kept, K = oracle.compact(mask, cu, b)
    return np.asarray(idx[:K]), np.asarray(cu_kept)


def test_matches_torch_sdpa_on_gathered_rows():
    torch = pytest.importorskip("torch")
    lengths, H, dh, b = [70, 33], 3, 8, 8
    q, k, v = _qkv(sum(lengths), H, dh, 1)
    idx, cu_kept = _kept(lengths, b, 2)
    got = oracle.attention_kept(q, k, v, idx, cu_kept, H, dh)
    for s in range(len(lengths)):
        rows = idx[cu_kept[s]:cu_kept[s + 1]]
        if len(rows) == 0:
            continue
        t = lambda a: torch.tensor(oracle.bf16_bits_to_f64(a[rows]).reshape(-1, H, dh)  # noqa
                                   .transpose(1, 0, 2))
        ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True)
        ref = ref.numpy().transpose(1, 0, 2).reshape(len(rows), H * dh)
        np.testing.assert_allclose(got[cu_kept[s]:cu_kept[s + 1]], ref, rtol=1e-12, atol=1e-14)


def test_pure_python_softmax_on_tiny_input():
    H, dh = 2, 2
    q, k, v = _qkv(6, H, dh, 3, scale=2.0)
    idx = np.array([0, 2, 3, 5])
    cu_kept = np.array([0, 4])
    got = oracle.attention_kept(q, k, v, idx, cu_kept, H, dh, scale=0.7)
    qf, kf, vf = (oracle.bf16_bits_to_f64(a) for a in (q, k, v))
    for r, i in enumerate(idx):
        for h in range(H):
            keys = [j for j in idx if j <= i]
            logits = [0.7 * sum(qf[i, h * dh + c] * kf[j, h * dh + c] for c in range(dh))
                      for j in keys]
            m = max(logits)
            w = [math.exp(x - m) for x in logits]
            z = sum(w)
            for c in range(dh):
                want = sum(wj / z * vf[j, h * dh + c] for wj, j in zip(w, keys))
                assert got[r, h * dh + c] == pytest.approx(want, rel=1e-13, abs=1e-15)


def test_constant_values_give_the_constant():
    L, H, dh = 40, 2, 4
    q, k, _ = _qkv(L, H, dh, 4)
    v = np.tile(synth.to_bf16_bits(np.array([[1.5, -2.0, 0.25, 3.0, 7.0, 0.0, -1.0, 0.5]])),
                (L, 1))
    idx, cu_kept = np.array([1, 2, 3, 10, 11, 30]), np.array([0, 6])
    got = oracle.attention_kept(q, k, v, idx, cu_kept, H, dh)
    np.testing.assert_allclose(got, np.tile(oracle.bf16_bits_to_f64(v[:1]), (6, 1)), rtol=1e-14)


def test_zero_queries_average_the_kept_prefix():
    L, H, dh = 30, 1, 3
    _, k, v = _qkv(L, H, dh, 5)
    q = np.zeros_like(k)
    idx, cu_kept = np.array([0, 4, 5, 6, 20, 29]), np.array([0, 6])
    got = oracle.attention_kept(q, k, v, idx, cu_kept, H, dh)
    vf = oracle.bf16_bits_to_f64(v)
    for r in range(6):
        np.testing.assert_allclose(got[r], vf[idx[:r + 1]].mean(axis=0), rtol=1e-13)


def test_keeping_everything_is_plain_causal_attention():
    L, H, dh = 25, 2, 4
    q, k, v = _qkv(L, H, dh, 6)
    got = oracle.attention_kept(q, k, v, np.arange(L), np.array([0, L]), H, dh)
    qf, kf, vf = (oracle.bf16_bits_to_f64(a).reshape(L, H, dh) for a in (q, k, v))
    for h in range(H):
        s = qf[:, h] @ kf[:, h].T / math.sqrt(dh)
        s[np.triu_indices(L, 1)] = -np.inf
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        np.testing.assert_allclose(got[:, h * dh:(h + 1) * dh], p @ vf[:, h], rtol=1e-12)


def test_sequences_do_not_attend_to_each_other():
    lengths, H, dh = [20, 20], 1, 4
    q, k, v = _qkv(40, H, dh, 7)
    idx = np.array([0, 1, 2, 25, 26])
    both = oracle.attention_kept(q, k, v, idx, np.array([0, 3, 5]), H, dh)
    second = oracle.attention_kept(q, k, v, idx[3:], np.array([0, 2]), H, dh)
    np.testing.assert_allclose(both[3:], second, rtol=1e-15)
    # as one sequence, the later rows would see the earlier ones
    merged = oracle.attention_kept(q, k, v, idx, np.array([0, 5]), H, dh)
    assert not np.allclose(merged[3:], second)


def test_residual_touches_only_kept_rows():
    x = synth.normal_bf16(10, 8, 0, 1)
    o = np.arange(24, dtype=np.float64).reshape(3, 8)
    idx = np.array([1, 4, 9])
    ex = oracle.attention_residual_exact(x, o, idx)
    xf = oracle.bf16_bits_to_f64(x)
    others = [i for i in range(10) if i not in idx]
    assert np.array_equal(ex[others], xf[others])
    np.testing.assert_array_equal(ex[idx], xf[idx] + o)


def test_rows_helper_equals_full_definition():
    lengths, H, dh, b = [90, 50], 2, 4, 8
    q, k, v = _qkv(sum(lengths), H, dh, 8)
    idx, cu_kept = _kept(lengths, b, 9)
    full = oracle.attention_kept(q, k, v, idx, cu_kept, H, dh)
    rows = [0, 1, int(cu_kept[1]) - 1, int(cu_kept[1]), len(idx) - 1]
    got = oracle.attention_kept_rows(q, k, v, idx, cu_kept, H, dh, rows)
    np.testing.assert_allclose(got, full[rows], rtol=1e-12, atol=1e-15)

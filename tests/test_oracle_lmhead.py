"""Pins of the oracle's lm-head loss (segment-based peak cutting extension).

The oracle restates mean next-token cross entropy and its gradients.  It is
checked against things other than itself: torch's fp64 cross entropy and
autograd (a library routine of the same definition), central finite
differences of its own loss (the gradient formula is not used), closed forms
(all-zero weights, two-class logistic loss), and invariants (a shared shift
of all logits of a token, ignored tokens acting as removed rows).
"""

import math

import numpy as np
import pytest

import oracle
from contextual_token_sparsity_b200 import synth


def _case(T, d, V, seed, ignore_frac=0.0, scale=1.0):
    rng = np.random.default_rng(seed)
    h = synth.to_bf16_bits(rng.standard_normal((T, d)))
    w = synth.to_bf16_bits(rng.standard_normal((V, d)) * scale / math.sqrt(d))
    y = rng.integers(0, V, size=T).astype(np.int32)
    y[rng.random(T) < ignore_frac] = -100
    return h, w, y


def test_matches_torch_cross_entropy_and_autograd():
    torch = pytest.importorskip("torch")
    h, w, y = _case(37, 24, 53, 1, ignore_frac=0.2, scale=3.0)
    loss, dh, dw, lse = oracle.lm_head_loss(h, w, y)
    ht = torch.tensor(oracle.bf16_bits_to_f64(h), requires_grad=True)
    wt = torch.tensor(oracle.bf16_bits_to_f64(w), requires_grad=True)
    z = ht @ wt.T
    ref = torch.nn.functional.cross_entropy(z, torch.tensor(y, dtype=torch.int64),
                                            ignore_index=-100, reduction="mean")
    ref.backward()
    assert loss == pytest.approx(ref.item(), rel=1e-13)
    np.testing.assert_allclose(dh, ht.grad.numpy(), rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(dw, wt.grad.numpy(), rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(lse, torch.logsumexp(z, 1).detach().numpy(), rtol=1e-14)


def test_gradients_match_central_differences():
    rng = np.random.default_rng(3)
    T, d, V = 6, 5, 7
    h = rng.standard_normal((T, d))
    w = rng.standard_normal((V, d))
    y = rng.integers(0, V, size=T)
    y[2] = -100
    _, dh, dw, _ = oracle.lm_head_loss_f64(h, w, y)
    eps = 1e-6
    for (t, c) in [(0, 0), (1, 3), (2, 1), (5, 4)]:
        hp, hm = h.copy(), h.copy()
        hp[t, c] += eps
        hm[t, c] -= eps
        fd = (oracle.lm_head_loss_f64(hp, w, y)[0] - oracle.lm_head_loss_f64(hm, w, y)[0]) / (2 * eps)
        assert dh[t, c] == pytest.approx(fd, abs=1e-8)
    for (v, c) in [(0, 0), (3, 2), (6, 4), (int(y[0]), 1)]:
        wp, wm = w.copy(), w.copy()
        wp[v, c] += eps
        wm[v, c] -= eps
        fd = (oracle.lm_head_loss_f64(h, wp, y)[0] - oracle.lm_head_loss_f64(h, wm, y)[0]) / (2 * eps)
        assert dw[v, c] == pytest.approx(fd, abs=1e-8)
    # the ignored token's row has no gradient
    assert np.all(dh[2] == 0.0)


def test_zero_weights_closed_form():
    T, d, V = 5, 3, 11
    rng = np.random.default_rng(4)
    h = rng.standard_normal((T, d))
    w = np.zeros((V, d))
    y = np.array([0, 4, -100, 10, 4])
    loss, dh, dw, lse = oracle.lm_head_loss_f64(h, w, y)
    n = 4
    assert loss == pytest.approx(math.log(V), rel=1e-15)
    np.testing.assert_allclose(lse, np.full(T, math.log(V)), rtol=1e-15)
    assert np.all(dh == 0.0)
    want = np.zeros((V, d))
    for t in range(T):
        if y[t] == -100:
            continue
        for v in range(V):
            want[v] += ((1.0 / V) - (1.0 if v == y[t] else 0.0)) / n * h[t]
    np.testing.assert_allclose(dw, want, rtol=1e-13, atol=1e-16)


def test_two_class_logistic_closed_form():
    # V = 2: the loss is softplus(z_other - z_target), its gradient the logistic
    h = np.array([[1.0], [-2.0], [0.5]])
    w = np.array([[1.5], [-0.25]])
    y = np.array([0, 1, 1])
    loss, dh, _, _ = oracle.lm_head_loss_f64(h, w, y)
    want, wdh = 0.0, []
    for t in range(3):
        z = [h[t, 0] * w[0, 0], h[t, 0] * w[1, 0]]
        m = z[1 - y[t]] - z[y[t]]
        want += math.log1p(math.exp(m))
        sig = 1.0 / (1.0 + math.exp(-m))
        # d/dh of softplus(h (w_o - w_y)) = sig * (w_o - w_y)
        wdh.append(sig * (w[1 - y[t], 0] - w[y[t], 0]) / 3)
    assert loss == pytest.approx(want / 3, rel=1e-14)
    np.testing.assert_allclose(dh[:, 0], wdh, rtol=1e-13)


def test_shared_logit_shift_is_invisible():
    # adding one vector u to every weight row adds h_t.u to every logit of
    # token t: softmax, loss and dh (rows of dz sum to 0) do not change
    h, w, y = _case(9, 8, 13, 6)
    u = np.array([0.5, -1.0, 0.25, 2.0, 0.0, -0.5, 1.0, 0.125])
    wf = oracle.bf16_bits_to_f64(w)
    hf = oracle.bf16_bits_to_f64(h)
    a = oracle.lm_head_loss_f64(hf, wf, y)
    b = oracle.lm_head_loss_f64(hf, wf + u[None, :], y)
    assert b[0] == pytest.approx(a[0], rel=1e-12)
    np.testing.assert_allclose(b[1], a[1], rtol=1e-9, atol=1e-13)


def test_ignored_tokens_act_as_removed_rows():
    h, w, y = _case(12, 6, 9, 7)
    y2 = y.copy()
    y2[[1, 5, 6]] = -100
    keep = [t for t in range(12) if t not in (1, 5, 6)]
    a = oracle.lm_head_loss(h, w, y2)
    b = oracle.lm_head_loss(h[keep], w, y[keep])
    assert a[0] == pytest.approx(b[0], rel=1e-14)
    np.testing.assert_allclose(a[1][keep], b[1], rtol=1e-14)
    np.testing.assert_allclose(a[2], b[2], rtol=1e-12, atol=1e-16)
    # all ignored: zero loss and gradients
    z = oracle.lm_head_loss(h, w, np.full(12, -100))
    assert z[0] == 0.0 and not z[1].any() and not z[2].any()


def test_out_of_range_target_rejected():
    h, w, y = _case(3, 4, 5, 8)
    y[1] = 5
    with pytest.raises(ValueError):
        oracle.lm_head_loss(h, w, y)


def test_rows_helper_equals_full_definition():
    h, w, y = _case(20, 16, 31, 9, ignore_frac=0.25)
    loss, dh, _, lse = oracle.lm_head_loss(h, w, y)
    n = int((y != -100).sum())
    rows = [0, 3, 7, 19]
    terms, dh_rows = oracle.lm_head_rows(h, w, y, rows, n)
    np.testing.assert_allclose(dh_rows, dh[rows], rtol=1e-12, atol=1e-16)
    full_terms, _ = oracle.lm_head_rows(h, w, y, range(20), n)
    assert full_terms.sum() / n == pytest.approx(loss, rel=1e-13)

"""GPU parity of the whole path (score -> select -> gather -> scatter) against
the CPU oracle, through the C ABI, on seeded synthetic inputs.

Bar: block maxima and block scores within 1e-2 relative; the keep mask
bit-exact outside a 1e-2 band around the threshold (and equal to the
kernel's own fp32 comparison everywhere); kept ids, per-sequence offsets,
kept count, gathered buffer and updated residual bit-exact given the mask.
"""

import numpy as np
import pytest

import oracle
from contextual_token_sparsity_b200 import lemo, synth
from contextual_token_sparsity_b200.pipeline import Layer, to_device_bf16, to_host_bits
from gpu_common import (assert_scores_close, check_all, check_mask, check_movement,
                        run_layer)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    torch.cuda.set_device(0)
    lemo.lemo_set_test_hooks(-1, 0)
    assert lemo.lemo_get_error() == lemo.LEMO_OK


def _inputs(lengths, H, dh, d, seed, frac=0.1):
    q, k, cu, _ = synth.qk_direct(lengths, H, dh, [frac] * len(lengths), seed)
    x = synth.normal_bf16(sum(lengths), d, seed, 7)
    y = synth.normal_bf16(sum(lengths), d, seed, 8)
    return q, k, cu, x, y


# Small cases: several tiles, ragged tails, empty and one-token sequences,
# both block sizes and head dims, more tiles than SMs (persistent loop).
SMALL = [
    ([700], 3, 128, 64, 64),
    ([300, 0, 1, 517, 64, 129], 2, 64, 128, 128),
    ([1000], 4, 64, 64, 40),
    ([257, 1025], 5, 128, 128, 24),
    ([4096], 2, 64, 64, 16),            # 272 tiles > 148 SMs
    ([1, 2, 3, 127, 128, 129, 255, 256, 383], 1, 64, 64, 8),
]


@pytest.mark.parametrize("lengths,H,dh,b,d", SMALL, ids=[str(c[0])[:30] for c in SMALL])
def test_small_shapes_match_oracle(lengths, H, dh, b, d):
    q, k, cu, x, y = _inputs(lengths, H, dh, d, seed=sum(lengths) % 97)
    s_ref = oracle.column_scores(oracle.score_blocks(q, k, cu, H, dh, b))
    theta = oracle.threshold_for_keep_ratio(s_ref, 0.5)
    res = run_layer(lengths, H, dh, b, d, q, k, x, y, theta)
    check_all(res, q, k, cu, H, dh, b, x, y, theta)


def test_all_ones_closed_form_exact():
    """Q = K = 1: every valid block max is exactly dh, empty blocks 0."""
    lengths, H, dh, b, d = [385, 129], 3, 128, 64, 8
    total = sum(lengths)
    ones = synth.to_bf16_bits(np.ones((total, H * dh)))
    x = synth.normal_bf16(total, d, 1, 7)
    res = run_layer(lengths, H, dh, b, d, ones, ones, x, x, theta=1.0)
    for L, M in zip(lengths, res["M"]):
        nb = -(-L // b)
        last = L - (nb - 1) * b
        for n in range(nb):
            for m in range(n + 1):
                empty = n == m and (b if n < nb - 1 else last) < 2
                assert M[n, m] == (0.0 if empty else float(dh)), (L, n, m, M[n, m])


def test_scale_is_positive_homogeneous():
    lengths, H, dh, b, d = [600], 2, 128, 64, 8
    q, k, cu, x, y = _inputs(lengths, H, dh, d, seed=5)
    r1 = run_layer(lengths, H, dh, b, d, q, k, x, y, theta=0.0)
    r2 = run_layer(lengths, H, dh, b, d, q, k, x, y, theta=0.0, scale=0.125)
    np.testing.assert_allclose(r2["scores"], 0.125 * r1["scores"], rtol=1e-6)
    s_ref = oracle.column_scores(oracle.score_blocks(q, k, cu, H, dh, b, scale=0.125))
    assert_scores_close(r2["scores"], s_ref)


def test_deterministic_bytes():
    lengths, H, dh, b, d = [2000, 300], 4, 128, 64, 64
    q, k, cu, x, y = _inputs(lengths, H, dh, d, seed=9)
    a = run_layer(lengths, H, dh, b, d, q, k, x, y, theta=1.0)
    c = run_layer(lengths, H, dh, b, d, q, k, x, y, theta=1.0)
    assert a["scores"].tobytes() == c["scores"].tobytes()
    for ma, mc in zip(a["M"], c["M"]):
        low = np.tril(np.ones_like(ma, dtype=bool))
        assert ma[low].tobytes() == mc[low].tobytes()


@pytest.mark.parametrize("theta,expect", [(-np.inf, "all"), (np.inf, "none")])
def test_keep_all_and_none(theta, expect):
    lengths, H, dh, b, d = [333, 200], 2, 64, 64, 16
    q, k, cu, x, y = _inputs(lengths, H, dh, d, seed=11)
    res = run_layer(lengths, H, dh, b, d, q, k, x, y, theta=theta)
    total = sum(lengths)
    if expect == "all":
        assert res["K"] == total and np.array_equal(res["kept_idx"], np.arange(total))
    else:
        assert res["K"] == 0 and (res["cu_kept"] == 0).all()
        assert np.array_equal(res["x"], x)
    check_movement(res, cu, b, x, y, 128)


def test_small_1k_full():
    """Single layer L=1024, d=512, H=8, dh=64, b=64, projected Q/K, 50th pct."""
    w = synth.WORKLOADS["small-1k"]
    inp = synth.make_workload("small-1k")
    cu = inp["cu_seqlens"]
    s_ref = oracle.column_scores(oracle.score_blocks(inp["q"], inp["k"], cu, w.H, w.dh, w.block))
    theta = oracle.threshold_for_keep_ratio(s_ref, 0.5)
    assert theta == pytest.approx(float(np.percentile(s_ref, 50)))
    res = run_layer(w.lengths, w.H, w.dh, w.block, w.d, inp["q"], inp["k"], inp["x"],
                    inp["y_out"], theta)
    check_all(res, inp["q"], inp["k"], cu, w.H, w.dh, w.block, inp["x"], inp["y_out"], theta)
    assert int(res["mask"].sum()) == 8


def test_many_short_sequences():
    """1500 sequences (empty, shorter than a block, a block and a token,
    a few blocks): the plan's prefix loop runs in two chunks and every
    kernel maps tiles, blocks and rows to their sequences by search."""
    rng = np.random.default_rng(21)
    lengths = [int(v) for v in rng.choice([0, 1, 5, 63, 64, 65, 130, 200], size=1500)]
    H, dh, b, d = 2, 64, 64, 16
    q, k, cu, x, y = _inputs(lengths, H, dh, d, seed=21)
    s_ref = oracle.column_scores(oracle.score_blocks(q, k, cu, H, dh, b))
    theta = oracle.threshold_for_keep_ratio(s_ref, 0.5)
    res = run_layer(lengths, H, dh, b, d, q, k, x, y, theta)
    check_all(res, q, k, cu, H, dh, b, x, y, theta)


def test_varlen_packing_equals_separate_calls():
    """A packed batch gives the same scores as each sequence on its own."""
    lengths, H, dh, b, d = [512, 130, 700], 2, 128, 64, 8
    q, k, cu, x, y = _inputs(lengths, H, dh, d, seed=13)
    packed = run_layer(lengths, H, dh, b, d, q, k, x, y, theta=0.0)["scores"]
    parts = []
    for s, L in enumerate(lengths):
        sl = slice(cu[s], cu[s + 1])
        parts.append(run_layer([L], H, dh, b, d, q[sl], k[sl], x[sl], y[sl], theta=0.0)["scores"])
    assert packed.tobytes() == np.concatenate(parts).tobytes()


# --------------------------------------------------------------------- errors

def test_invalid_cu_seqlens_reported_on_device():
    import torch
    layer = Layer([256], 2, 64, 64, 8, keep_block_max=True)
    bad = torch.tensor([0, 300], dtype=torch.int32, device="cuda")  # cu[batch] != total_L
    layer.shape.cu_seqlens = bad.data_ptr()
    q = to_device_bf16(synth.to_bf16_bits(np.ones((256, 128))))
    layer.block_scores.fill_(-7.0)
    layer.score(q, q)
    assert lemo.lemo_get_error() == lemo.LEMO_ERR_INVALID_ARG
    assert (layer.block_scores.cpu() == -7.0).all()  # nothing written
    assert lemo.lemo_get_error() == lemo.LEMO_OK       # cleared


def test_gather_capacity_and_index_checks():
    import torch
    x = torch.zeros((100, 16), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((64, 16), dtype=torch.bfloat16, device="cuda")
    idx = torch.arange(100, dtype=torch.int32, device="cuda")
    K = torch.tensor([100], dtype=torch.int32, device="cuda")
    lemo.lemo_gather_pad(x, idx, K, 128, y)            # needs 128 rows, has 64
    assert lemo.lemo_get_error() == lemo.LEMO_ERR_CAPACITY
    idx[5] = 1000                                      # out of range row
    K[0] = 10
    y2 = torch.zeros((128, 16), dtype=torch.bfloat16, device="cuda")
    lemo.lemo_gather_pad(x, idx, K, 128, y2)
    assert lemo.lemo_get_error() == lemo.LEMO_ERR_INVALID_ARG
    lemo.lemo_scatter_residual(x, y2, idx, K)
    assert lemo.lemo_get_error() == lemo.LEMO_ERR_INVALID_ARG


def test_select_bounded_wait_times_out_and_recovers():
    """One compaction tile withholds its descriptor: the tiles after it give up
    after the (shortened) bounded wait and report LEMO_ERR_TIMEOUT; K reads 0.
    The next call, without the hook, is correct."""
    lengths, H, dh, b, d = [9000], 1, 64, 64, 8
    q, k, cu, x, y = _inputs(lengths, H, dh, d, seed=17)
    layer = Layer(lengths, H, dh, b, d)
    layer.score(to_device_bf16(q), to_device_bf16(k))
    assert lemo.lemo_get_error() == lemo.LEMO_OK
    try:
        lemo.lemo_set_test_hooks(select_skip_publish_tile=1, spin_limit_ns=50_000_000)
        layer.select(0.0)
        assert lemo.lemo_get_error() == lemo.LEMO_ERR_TIMEOUT
        assert int(layer.kept_total.item()) == 0
    finally:
        lemo.lemo_set_test_hooks(-1, 0)
    layer.select(0.0)
    assert lemo.lemo_get_error() == lemo.LEMO_OK
    assert int(layer.kept_total.item()) == sum(lengths)

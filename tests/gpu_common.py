"""Shared helpers of the GPU parity tests: run one layer of the path through
the C ABI and compare every output with the CPU oracle."""

import numpy as np

import oracle
from contextual_token_sparsity_b200 import lemo
from contextual_token_sparsity_b200.pipeline import Layer, to_device_bf16, to_host_bits

SCORE_RTOL = 1e-2  # block scores: relative tolerance of the parity bar
BAND = 1e-2        # mask bits within this relative band of theta are exempt


def run_layer(lengths, H, dh, b, d, q, k, x, y_out, theta, scale=1.0, pad_to=128,
              keep_block_max=True):
    layer = Layer(lengths, H, dh, b, d, pad_to=pad_to, keep_block_max=keep_block_max)
    qd, kd = to_device_bf16(q), to_device_bf16(k)
    xd, yd = to_device_bf16(x), to_device_bf16(y_out)
    layer.step(qd, kd, theta, xd, yd, scale=scale)
    st = lemo.lemo_get_error()
    assert st == lemo.LEMO_OK, lemo.STATUS.get(st, st)
    K = int(layer.kept_total.item())
    res = {
        "layer": layer,
        "scores": layer.block_scores[: layer.total_blocks].cpu().numpy().astype(np.float64),
        "M": layer.block_max_list() if keep_block_max else None,
        "mask": layer.mask[: layer.total_blocks].cpu().numpy(),
        "K": K,
        "kept_idx": layer.kept_idx[:K].cpu().numpy(),
        "cu_kept": layer.cu_kept.cpu().numpy(),
        "y": to_host_bits(layer.y),
        "x": to_host_bits(xd),
    }
    return res


def assert_scores_close(got, want, what="scores"):
    want = np.asarray(want, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    floor = 1e-6 * max(1.0, float(np.abs(want).max()) if want.size else 1.0)
    err = np.abs(got - want)
    bad = err > SCORE_RTOL * np.abs(want) + floor
    assert not bad.any(), (what, int(bad.sum()), float((err / np.maximum(np.abs(want), 1e-30)).max()))
    return float((err / np.maximum(np.abs(want), floor)).max()) if want.size else 0.0


def check_mask(res, scores_ref, theta):
    """Mask bit-exact outside the tolerance band; inside, it must still be the
    kernel's own fp32 decision on its own scores."""
    mask = res["mask"]
    ref = oracle.keep_mask(scores_ref, theta)
    band = np.abs(scores_ref - theta) <= BAND * abs(theta) if np.isfinite(theta) else \
        np.zeros_like(ref, dtype=bool)
    assert np.array_equal(mask[~band], ref[~band])
    own = oracle.keep_mask(res["scores"].astype(np.float32), np.float32(theta))
    assert np.array_equal(mask, own)
    return int(band.sum())


def check_movement(res, cu, b, x, y_out, pad_to):
    """Compaction, gather and scatter bit-exact given the GPU's own mask."""
    idx_ref, cu_ref, K_ref = oracle.compact(res["mask"], cu, b)
    assert res["K"] == K_ref
    assert np.array_equal(res["kept_idx"], idx_ref)
    assert np.array_equal(res["cu_kept"], cu_ref)
    y_ref = oracle.gather_pad(x, idx_ref, pad_to)
    assert np.array_equal(res["y"][: y_ref.shape[0]], y_ref)
    x_ref = oracle.scatter_residual(x, y_out, idx_ref)
    assert np.array_equal(res["x"], x_ref)


def check_all(res, q, k, cu, H, dh, b, x, y_out, theta, scale=1.0, pad_to=128):
    M_ref = oracle.score_blocks(q, k, cu, H, dh, b, scale=scale)
    s_ref = oracle.column_scores(M_ref)
    if res["M"] is not None:
        for Mg, Mr in zip(res["M"], M_ref):
            low = np.tril(np.ones_like(Mr, dtype=bool))
            assert_scores_close(Mg[low], Mr[low], "block_max")
    err = assert_scores_close(res["scores"], s_ref)
    check_mask(res, s_ref, theta)
    check_movement(res, cu, b, x, y_out, pad_to)
    return s_ref, err

"""lemo_select_static_ws: token selection for callers that cannot allocate.

Some callers of this library cannot allocate device memory where they select
tokens (a memory pool that owns the whole GPU, or a loop that must not pay for
an allocation's synchronisation).  lemo_select_static_ws keeps its scratch in
a fixed array inside the library instead of a caller-provided workspace.
These tests call it through the C ABI and check that, on two calls in a row,
it returns exactly what lemo_select returns for the same inputs (the outputs
are integers and masks, so the comparison is exact).  The file is named so
that pytest collects it last.
"""

import numpy as np
import pytest

from contextual_token_sparsity_b200 import lemo, synth

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
    lemo.lemo_get_error()


def _outputs(layer_like, n_blocks, total_L, batch):
    import torch
    return {
        "mask": torch.full((max(n_blocks, 1),), 7, dtype=torch.uint8, device="cuda"),
        "kept_idx": torch.full((max(total_L, 1),), -1, dtype=torch.int32, device="cuda"),
        "cu_kept": torch.full((batch + 1,), -1, dtype=torch.int32, device="cuda"),
        "kept_total": torch.full((1,), -1, dtype=torch.int32, device="cuda"),
    }


def _host(o, n_blocks):
    K = int(o["kept_total"].item())
    return (o["mask"][:n_blocks].cpu().numpy(), K, o["kept_idx"][:K].cpu().numpy(),
            o["cu_kept"].cpu().numpy())


def test_static_workspace_select_matches_lemo_select_twice():
    from contextual_token_sparsity_b200.pipeline import Layer, to_device_bf16
    lengths, H, dh, b = [3000, 0, 777, 5000], 2, 64, 64
    q, k, cu, _ = synth.qk_direct(lengths, H, dh, [0.1] * len(lengths), seed=23)
    layer = Layer(lengths, H, dh, b, d=8)
    scores = layer.score(to_device_bf16(q), to_device_bf16(k)).clone()
    assert lemo.lemo_get_error() == lemo.LEMO_OK
    s = scores[: layer.total_blocks].cpu().numpy().astype(np.float64)
    thetas = [float(np.median(s)), float(np.quantile(s, 0.8))]
    for theta in thetas:  # two calls in a row, different thresholds
        ref = _outputs(layer, layer.total_blocks, layer.total_L, len(lengths))
        got = _outputs(layer, layer.total_blocks, layer.total_L, len(lengths))
        lemo.lemo_select(layer.shape, scores, theta, ref["mask"], ref["kept_idx"],
                         ref["cu_kept"], ref["kept_total"], layer.ws)
        lemo.lemo_select_static_ws(layer.shape, scores, theta, got["mask"], got["kept_idx"],
                                   got["cu_kept"], got["kept_total"])
        assert lemo.lemo_get_error() == lemo.LEMO_OK
        m_ref, K_ref, i_ref, c_ref = _host(ref, layer.total_blocks)
        m_got, K_got, i_got, c_got = _host(got, layer.total_blocks)
        assert K_got == K_ref > 0
        assert np.array_equal(m_got, m_ref)
        assert np.array_equal(i_got, i_ref)
        assert np.array_equal(c_got, c_ref)


def test_static_workspace_select_rejects_shapes_over_its_limit():
    import torch
    cu = torch.zeros(5002, dtype=torch.int32, device="cuda")
    scores = torch.zeros(8, dtype=torch.float32, device="cuda")
    out = torch.zeros(8, dtype=torch.int32, device="cuda")
    mask = torch.zeros(8, dtype=torch.uint8, device="cuda")
    too_many_sequences = lemo.lemo_shape(5001, cu.data_ptr(), 0, 0, 1, 64, 64)
    too_many_tokens = lemo.lemo_shape(1, cu.data_ptr(), (1 << 24) + 1, (1 << 22), 1, 64, 64)
    for shape in (too_many_sequences, too_many_tokens):
        with pytest.raises(lemo.LemoError) as e:
            lemo.lemo_select_static_ws(shape, scores, 0.0, mask, out, out, out)
        assert e.value.status == lemo.LEMO_ERR_CAPACITY
    assert lemo.lemo_get_error() == lemo.LEMO_OK  # nothing was enqueued


def _random_scores_layer(lengths, seed):
    """A Layer for `lengths` (block size 64) with seeded random block scores on
    the device; selection needs nothing else."""
    import torch
    from contextual_token_sparsity_b200.pipeline import Layer
    layer = Layer(lengths, 1, 64, 64, d=8)
    rng = np.random.default_rng(seed)
    s = rng.standard_normal(max(layer.total_blocks, 1)).astype(np.float32)
    layer.block_scores.copy_(torch.from_numpy(s))
    return layer, s[: layer.total_blocks].astype(np.float64)


def _compare_calls(layer, theta):
    batch = len(layer.lengths)
    ref = _outputs(layer, layer.total_blocks, layer.total_L, batch)
    got = _outputs(layer, layer.total_blocks, layer.total_L, batch)
    lemo.lemo_select(layer.shape, layer.block_scores, theta, ref["mask"], ref["kept_idx"],
                     ref["cu_kept"], ref["kept_total"], layer.ws)
    lemo.lemo_select_static_ws(layer.shape, layer.block_scores, theta, got["mask"],
                               got["kept_idx"], got["cu_kept"], got["kept_total"])
    assert lemo.lemo_get_error() == lemo.LEMO_OK
    m_ref, K_ref, i_ref, c_ref = _host(ref, layer.total_blocks)
    m_got, K_got, i_got, c_got = _host(got, layer.total_blocks)
    assert K_got == K_ref > 0
    assert np.array_equal(m_got, m_ref)
    assert np.array_equal(i_got, i_ref)
    assert np.array_equal(c_got, c_ref)


def test_static_workspace_select_at_its_documented_limits():
    """batch = 4096 sequences (some empty) holding exactly 2^24 tokens: the
    largest shape the fixed array is documented to hold (plan arrays of 4097
    entries and 8192 look-back descriptors)."""
    rng = np.random.default_rng(41)
    lengths = rng.integers(1, 8192, 4096)
    lengths[rng.choice(4096, 300, replace=False)] = 0
    lengths = np.floor(lengths * ((1 << 24) / lengths.sum())).astype(np.int64)
    lengths[np.argmax(lengths)] += (1 << 24) - int(lengths.sum())
    assert lengths.sum() == 1 << 24 and (lengths == 0).sum() >= 300
    layer, s = _random_scores_layer(lengths.tolist(), seed=42)
    for theta in (float(np.median(s)), float(np.quantile(s, 0.9))):  # two calls in a row
        _compare_calls(layer, theta)


def test_static_workspace_select_times_out_and_recovers():
    """A compaction tile withholds its look-back descriptor (test hook): the
    tiles after it give up after the shortened bounded wait, the call reports
    LEMO_ERR_TIMEOUT and leaves K = 0.  The next call on the same shared array
    matches lemo_select, so each call re-initialises the look-back state."""
    import torch
    layer, s = _random_scores_layer([9000, 5000], seed=43)
    kept_total = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    try:
        lemo.lemo_set_test_hooks(select_skip_publish_tile=1, spin_limit_ns=50_000_000)
        lemo.lemo_select_static_ws(layer.shape, layer.block_scores, float(np.min(s)),
                                   layer.mask, layer.kept_idx, layer.cu_kept, kept_total)
        assert lemo.lemo_get_error() == lemo.LEMO_ERR_TIMEOUT
        assert int(kept_total.item()) == 0
    finally:
        lemo.lemo_set_test_hooks(-1, 0)
    _compare_calls(layer, float(np.median(s)))

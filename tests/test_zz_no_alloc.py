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

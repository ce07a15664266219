"""GPU parity of the extensions beyond the forward path:

* backward token movement: input recomputation by subtraction (bit-exact
  against the oracle's one-rounding definition) and the gradient passes built
  from the forward gather / scatter kernels;
* MLP-block elimination: token and block scores from MLP activations (ReLU
  outputs, or SiLU(gate) * up) within 1e-2 of the oracle, then selection.
"""

import numpy as np
import pytest

import oracle
from contextual_token_sparsity_b200 import lemo, synth
from contextual_token_sparsity_b200.pipeline import Layer, to_device_bf16, to_host_bits
from gpu_common import assert_scores_close, check_mask

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


def _kept(lengths, b, mask_seed):
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    nb = sum(-(-L // b) for L in lengths)
    mask = np.random.default_rng(mask_seed).integers(0, 2, nb).astype(np.uint8)
    idx, cu_kept, K = oracle.compact(mask, cu, b)
    return idx, K


def test_recompute_input_round_trip():
    import torch
    lengths, b, d = [700, 129], 64, 256
    idx, K = _kept(lengths, b, 3)
    x_in = synth.normal_bf16(sum(lengths), d, 3, 7)
    y = synth.normal_bf16(K, d, 3, 8) if K else np.zeros((1, d), np.uint16)
    x_out = oracle.scatter_residual(x_in, y, idx)
    xd = to_device_bf16(x_out)
    yd = to_device_bf16(y)
    idx_d = torch.from_numpy(idx).cuda() if K else torch.zeros(1, dtype=torch.int32, device="cuda")
    K_d = torch.tensor([K], dtype=torch.int32, device="cuda")
    lemo.lemo_recompute_input(xd, yd, idx_d, K_d)
    assert lemo.lemo_get_error() == lemo.LEMO_OK
    assert np.array_equal(to_host_bits(xd), oracle.recompute_input(x_out, y, idx))


def test_backward_token_movement_from_forward_kernels():
    """dy_out = gather(dx) at the kept rows; dx_in = dx + scatter(dy_in)."""
    import torch
    lengths, b, d = [512, 300], 64, 128
    idx, K = _kept(lengths, b, 4)
    total = sum(lengths)
    dx = synth.normal_bf16(total, d, 4, 9)
    dy_in = synth.normal_bf16(K, d, 4, 10)
    layer_idx = torch.from_numpy(idx).cuda()
    K_d = torch.tensor([K], dtype=torch.int32, device="cuda")
    dxd = to_device_bf16(dx)
    dy_out = torch.empty((-(-K // 128) * 128, d), dtype=torch.bfloat16, device="cuda")
    lemo.lemo_gather_pad(dxd, layer_idx, K_d, 128, dy_out)
    lemo.lemo_scatter_residual(dxd, to_device_bf16(dy_in), layer_idx, K_d)
    assert lemo.lemo_get_error() == lemo.LEMO_OK
    assert np.array_equal(to_host_bits(dy_out), oracle.gather_pad(dx, idx, 128))
    assert np.array_equal(to_host_bits(dxd), oracle.scatter_residual(dx, dy_in, idx))


def _mlp_gpu(lengths, b, mats, gated):
    import torch
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    layer = Layer(lengths, 1, 64, b, d=8)
    tok = torch.full((sum(lengths),), float("nan"), dtype=torch.float32, device="cuda")
    dev = [to_device_bf16(m) for m in mats]
    if gated:
        lemo.lemo_mlp_block_scores(layer.shape, layer.block_scores, layer.ws, gate=dev[0], up=dev[1],
                                   token_scores=tok)
    else:
        lemo.lemo_mlp_block_scores(layer.shape, layer.block_scores, layer.ws, act=dev[0],
                                   token_scores=tok)
    assert lemo.lemo_get_error() == lemo.LEMO_OK
    return layer, tok.cpu().numpy().astype(np.float64), \
        layer.block_scores[: layer.total_blocks].cpu().numpy().astype(np.float64), cu


# 400 sequences of 0 to 200 tokens: every token row finds its sequence and block by search
MANY = [int(v) for v in np.random.default_rng(51).choice([0, 1, 63, 64, 65, 200], size=400)]


@pytest.mark.parametrize("gated", [False, True], ids=["relu", "silu-gated"])
@pytest.mark.parametrize("lengths,b,d_ff", [([300, 0, 517, 1], 64, 136), ([1000, 257], 128, 512),
                                            (MANY, 64, 64)])
def test_mlp_scores_match_oracle_and_select(lengths, b, d_ff, gated):
    mats = synth.mlp_activations(sum(lengths), d_ff, 0.1, seed=len(lengths), gated=gated)
    layer, tok, blk, cu = _mlp_gpu(lengths, b, mats, gated)
    want_tok = oracle.mlp_token_scores(gate_bits=mats[0], up_bits=mats[1]) if gated else \
        oracle.mlp_token_scores(act_bits=mats[0])
    want_blk = oracle.mlp_block_scores(want_tok, cu, b)
    assert_scores_close(tok, want_tok, "mlp token scores")
    assert_scores_close(blk, want_blk, "mlp block scores")
    theta = oracle.threshold_for_keep_ratio(want_blk, 0.5)
    layer.select(theta)
    assert lemo.lemo_get_error() == lemo.LEMO_OK
    res = {"mask": layer.mask[: layer.total_blocks].cpu().numpy(), "scores": blk}
    check_mask(res, want_blk, theta)
    idx_ref, cu_ref, K_ref = oracle.compact(res["mask"], cu, b)
    K = int(layer.kept_total.item())
    assert K == K_ref and np.array_equal(layer.kept_idx[:K].cpu().numpy(), idx_ref)


def test_mlp_scores_llama7b_shape():
    """L = 16384 tokens, d_ff = 11008 (Llama-2-7B MLP), SiLU-gated."""
    L, d_ff, b = 16384, 11008, 64
    gate, up = synth.mlp_activations(L, d_ff, 0.1, seed=0, gated=True)
    layer, tok, blk, cu = _mlp_gpu([L], b, (gate, up), True)
    want_tok = oracle.mlp_token_scores(gate_bits=gate, up_bits=up)
    assert_scores_close(tok, want_tok, "mlp token scores 16K")
    assert_scores_close(blk, oracle.mlp_block_scores(want_tok, cu, b), "mlp block scores 16K")


def test_mlp_scores_write_only_their_blocks():
    """A varlen batch whose block count is below the host-side bound: the
    entries after block_scores[total_blocks - 1] must keep their bytes."""
    import torch
    lengths, b, d_ff = [300, 0, 517, 1], 64, 64   # 15 blocks; the host bound is 16
    (act,) = synth.mlp_activations(sum(lengths), d_ff, 0.1, seed=1, gated=False)
    layer = Layer(lengths, 1, 64, b, d=8)
    assert layer.total_blocks == 15
    buf = torch.full((layer.total_blocks + 8,), -3.0, dtype=torch.float32, device="cuda")
    lemo.lemo_mlp_block_scores(layer.shape, buf[: layer.total_blocks], layer.ws,
                               act=to_device_bf16(act))
    assert lemo.lemo_get_error() == lemo.LEMO_OK
    out = buf.cpu().numpy()
    assert (out[layer.total_blocks:] == -3.0).all()
    assert (out[: layer.total_blocks] >= 0).all()

"""GPU parity of the segmented lm-head loss (segment-based peak cutting).

The library computes logits in fp32 from bf16 inputs, rounds the logit
gradient dz and the hidden-state gradient dh to bf16 and accumulates dW in
fp32.  Tolerances, from that arithmetic (u = 2^-8, twice bf16's unit
roundoff):

* per-token loss terms and the loss: fp32 logits of d-term sums and an fp32
  log-sum-exp, |error| <= 1e-4 absolute per token at d <= 4096 (observed
  ~1e-6); the loss within 1e-5 relative.
* dh_t = dz_t W: rounding dz to bf16 moves each term by at most u/2 |dz_tv|,
  and sum_v |dz_tv| <= 2/n, so |error_tc| <= u (2/n) max_v |W_vc| plus the
  output rounding u |dh_tc|.
* dW_v = sum_t dz_tv h_t: |error_vc| <= u sum_t |dz_tv| |h_tc| (+ fp32 sums).

Segmenting must not change the result beyond those bounds, at any segment
size, including a ragged last segment.
"""

import numpy as np
import pytest

import oracle
from contextual_token_sparsity_b200 import lemo, synth

pytestmark = pytest.mark.gpu
U = 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    torch.cuda.set_device(0)
    lemo.lemo_set_test_hooks(-1, 0)


def _bf16_dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


def run(h, w, y, seg_rows, want_dh=True, want_dw=True, dw_init=None, ignore_index=-100):
    import torch
    T, d = h.shape
    V = w.shape[0]
    hd, wd = _bf16_dev(h), _bf16_dev(w)
    yd = torch.from_numpy(np.asarray(y, dtype=np.int32)).cuda()
    loss = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    tl = torch.full((max(T, 1),), float("nan"), dtype=torch.float32, device="cuda")
    dh = torch.full((max(T, 1), d), -1, dtype=torch.int16, device="cuda") if want_dh else None
    dw = None
    if want_dw:
        dw = (torch.zeros((V, d), dtype=torch.float32, device="cuda") if dw_init is None
              else torch.from_numpy(np.asarray(dw_init, dtype=np.float32)).cuda())
    ws = torch.empty(lemo.lemo_segment_loss_workspace_size(T, V, seg_rows), dtype=torch.uint8,
                     device="cuda")
    lemo.lemo_segment_loss(hd, wd, yd, seg_rows, loss, ws, token_loss=tl, dh=dh, dw=dw,
                           ignore_index=ignore_index)
    st = lemo.lemo_get_error()
    out = {"status": st, "loss": float(loss.item()), "token_loss": tl[:T].cpu().numpy()}
    if want_dh:
        out["dh"] = oracle.bf16_bits_to_f64(dh[:T].cpu().numpy().view(np.uint16))
    if want_dw:
        out["dw"] = dw.cpu().numpy().astype(np.float64)
    return out


def check_against_oracle(got, h, w, y, ignore_index=-100):
    loss, dh, dw, lse = oracle.lm_head_loss(h, w, y, ignore_index)
    hf, wf = oracle.bf16_bits_to_f64(h), oracle.bf16_bits_to_f64(w)
    valid = np.asarray(y) != ignore_index
    n = int(valid.sum())
    z = hf @ wf.T
    terms = np.where(valid, lse - z[np.arange(len(y)), np.where(valid, y, 0)], 0.0)
    assert np.abs(got["token_loss"] - terms).max() <= 1e-4
    assert got["loss"] == pytest.approx(loss, rel=1e-5, abs=1e-6)
    if n == 0:
        return
    tol_dh = U * (2.0 / n) * np.abs(wf).max(axis=0)[None, :] + U * np.abs(dh) + 1e-30
    assert np.all(np.abs(got["dh"] - dh) <= tol_dh), float((np.abs(got["dh"] - dh) / tol_dh).max())
    if "dw" in got:
        p = np.exp(z - lse[:, None])
        p[np.nonzero(valid)[0], np.asarray(y)[valid]] -= 1.0
        p[~valid] = 0.0
        absdz = np.abs(p) / n
        tol_dw = U * (absdz.T @ np.abs(hf)) + 1e-6 * np.abs(dw).max()
        assert np.all(np.abs(got["dw"] - dw) <= tol_dw), float((np.abs(got["dw"] - dw) / tol_dw).max())


@pytest.mark.parametrize("T,d,V,seg,ign", [(300, 64, 1000, 64, 0.1), (50, 32, 77, 7, 0.0),
                                           (129, 128, 4099, 128, 0.3), (1, 8, 5, 1, 0.0)],
                         ids=["ragged-tail", "odd-vocab", "vocab-tail", "single-token"])
def test_matches_oracle(T, d, V, seg, ign):
    h, w, y = synth.lm_head_inputs(T, d, V, seed=T + V, ignore_frac=ign)
    got = run(h, w, y, seg)
    assert got["status"] == lemo.LEMO_OK
    check_against_oracle(got, h, w, y)


def test_segment_size_does_not_change_the_result():
    h, w, y = synth.lm_head_inputs(200, 64, 517, seed=11, ignore_frac=0.1)
    for seg in (1, 3, 64, 199, 200, 4096):
        got = run(h, w, y, seg)
        assert got["status"] == lemo.LEMO_OK
        check_against_oracle(got, h, w, y)


def test_mid_size_several_segments():
    # 2048 tokens in segments of 384: five full segments and a ragged one
    h, w, y = synth.lm_head_inputs(2048, 512, 4096, seed=5, ignore_frac=0.05)
    got = run(h, w, y, 384)
    assert got["status"] == lemo.LEMO_OK
    check_against_oracle(got, h, w, y)


def test_all_ignored_and_empty():
    h, w, y = synth.lm_head_inputs(40, 16, 33, seed=2)
    y[:] = -100
    init = np.random.default_rng(0).standard_normal((33, 16)).astype(np.float32)
    got = run(h, w, y, 16, dw_init=init)
    assert got["status"] == lemo.LEMO_OK
    assert got["loss"] == 0.0 and np.all(got["token_loss"] == 0.0)
    assert np.all(got["dh"] == 0.0)
    assert np.array_equal(got["dw"], init.astype(np.float64))   # nothing accumulated
    got = run(h[:0], w, y[:0], 16)
    assert got["status"] == lemo.LEMO_OK and got["loss"] == 0.0


def test_custom_ignore_index_and_bad_target():
    h, w, y = synth.lm_head_inputs(64, 16, 50, seed=3)
    y2 = y.copy()
    y2[[3, 9]] = 7777          # the caller's ignore index
    got = run(h, w, y2, 16, ignore_index=7777)
    assert got["status"] == lemo.LEMO_OK
    check_against_oracle(got, h, w, y2, ignore_index=7777)
    y3 = y.copy()
    y3[5] = 50                 # outside [0, V): reported, adds nothing
    got = run(h, w, y3, 16)
    assert got["status"] == lemo.LEMO_ERR_INVALID_ARG
    assert got["token_loss"][5] == 0.0
    y4 = y.copy()
    y4[5] = -100
    check_against_oracle({k: v for k, v in got.items() if k != "status"}, h, w, y4)


def test_dw_accumulates_and_frozen_head():
    h, w, y = synth.lm_head_inputs(96, 32, 100, seed=4)
    once = run(h, w, y, 32)
    twice = run(h, w, y, 32, dw_init=once["dw"])
    np.testing.assert_allclose(twice["dw"], 2 * once["dw"], rtol=1e-6, atol=1e-9)
    frozen = run(h, w, y, 32, want_dw=False)
    assert frozen["loss"] == once["loss"]
    assert np.array_equal(frozen["dh"], once["dh"])


def test_lmhead_7b_workload_sampled_rows():
    """Llama-2-7B head over 16384 tokens in 16 segments: sampled token rows
    against the oracle row by row, the loss against the mean of the token
    terms, and sum_v dW[v, :] = 0 (rows of dz sum to zero)."""
    cfg = synth.LM_HEAD_WORKLOADS["lmhead-llama7b-16k"]
    T, d, V, S = cfg["T"], cfg["d"], cfg["V"], cfg["seg_rows"]
    h, w, y = synth.lm_head_inputs(T, d, V, cfg["seed"])
    got = run(h, w, y, S)
    assert got["status"] == lemo.LEMO_OK
    rows = [0, 1, 1023, 1024, 5000, 8191, 12345, T - 1]
    terms, dh_rows = oracle.lm_head_rows(h, w, y, rows, T)
    assert np.abs(got["token_loss"][rows] - terms).max() <= 1e-4
    wf_absmax = np.abs(oracle.bf16_bits_to_f64(w)).max(axis=0)
    tol = U * (2.0 / T) * wf_absmax[None, :] + U * np.abs(dh_rows)
    assert np.all(np.abs(got["dh"][rows] - dh_rows) <= tol)
    assert got["loss"] == pytest.approx(float(got["token_loss"].astype(np.float64).mean()), rel=1e-6)
    colsum = got["dw"].sum(axis=0)
    # each |dz| entry is off by at most u/2 of itself; sum_t sum_v |dz_tv| |h_tc| <= 2 max|h|
    bound = U * 2.0 * np.abs(oracle.bf16_bits_to_f64(h)).max(axis=0) + 1e-5
    assert np.all(np.abs(colsum) <= bound)
    # the activation peak is one segment's fp32 logits, four segments' bf16
    # gradients (dW is accumulated once per four segments) and the logit
    # rows' softmax partials (8 bytes per 128 columns): (12 V + 16 ntiles) S
    # bytes, against (6 V + 16 ntiles) T unsegmented, about 8x smaller at 16
    # segments
    ntiles = -(-V // 256)
    seg = lemo.lemo_segment_loss_workspace_size(T, V, S)
    full = lemo.lemo_segment_loss_workspace_size(T, V, T)
    fixed = lemo.lemo_segment_loss_workspace_size(T, V, 1) - (12 * V + 16 * ntiles)
    want = (6 * V + 16 * ntiles) * T / ((12 * V + 16 * ntiles) * S)
    assert (full - fixed) / (seg - fixed) == pytest.approx(want, rel=1e-3)
    assert want > 7.9

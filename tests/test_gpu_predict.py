"""GPU parity of the predictor path (step a8) against the CPU oracle.

Predicted block scores within 1e-2 relative of the oracle's float64
evaluation (the kernels compute in fp32, so the observed error is ~1e-6);
pruned neurons left out of compacted weights give the same scores; at the
Llama-2-13B workload the scores match the stored oracle values and the
predicted keep mask equals the oracle's outside the tolerance band, so the
recall against the exact mask is the stored one.
"""

import json
import os

import numpy as np
import pytest

import oracle
from contextual_token_sparsity_b200 import lemo, synth
from gpu_common import BAND, assert_scores_close

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    torch.cuda.set_device(0)
    lemo.lemo_set_test_hooks(-1, 0)


def _dev(bits):
    from contextual_token_sparsity_b200.pipeline import to_device_bf16
    return to_device_bf16(bits)


def _dev_misaligned(bits):
    """Device copy whose data pointer is 2 bytes past a 256-byte boundary."""
    import torch
    flat = np.zeros(bits.size + 1, np.uint16)
    flat[1:] = np.ascontiguousarray(bits).ravel()
    t = torch.from_numpy(flat.view(np.int16)).cuda()
    return t[1:].view(bits.shape)


def run_predict(lengths, H, dh, b, x_bits, w1q, w2q, w1k, w2k, misaligned=False):
    import torch
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    cu_d = torch.from_numpy(cu).cuda()
    shape = lemo.make_shape(cu_d, int(cu[-1]), max(lengths), H, dh, b)
    d, rank = x_bits.shape[1], w1q.shape[1]
    ws = torch.empty(lemo.lemo_predict_workspace_size(shape, d, rank), dtype=torch.uint8,
                     device="cuda")
    nblk = sum(-(-L // b) for L in lengths)
    out = torch.full((max(nblk, 1),), float("nan"), dtype=torch.float32, device="cuda")
    wdev = _dev_misaligned if misaligned else _dev
    lemo.lemo_predict_scores(shape, _dev(x_bits), wdev(w1q), wdev(w2q), wdev(w1k), wdev(w2k),
                             out, ws)
    st = lemo.lemo_get_error()
    assert st == lemo.LEMO_OK, lemo.STATUS.get(st, st)
    return out[:nblk].cpu().numpy().astype(np.float64), cu


def oracle_predict(lengths, H, dh, b, x_bits, w1q, w2q, w1k, w2k):
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    reps = oracle.block_representatives(x_bits, cu, b)
    qh = oracle.predictor_embeddings(reps, w1q, w2q)
    kh = oracle.predictor_embeddings(reps, w1k, w2k)
    return oracle.predict_scores(qh, kh, cu, b, H, dh)[1]


CASES = [([300, 0, 517, 64, 1], 2, 64, 64, 64, 48),
         ([1000], 3, 128, 128, 256, 40),
         ([2049, 640], 4, 32, 64, 136, 100),   # rank % 8 != 0: W1 copied into padded planes
         ([700, 130], 3, 20, 64, 64, 37),       # odd rank and dh % 8 != 0: padded weight copies
         ([513], 2, 24, 128, 40, 6),
         ([777], 2, 64, 64, 64, 24)]            # one sequence, b = 64: the pooling pass writes the plan


@pytest.mark.parametrize("lengths,H,dh,b,d,rank", CASES, ids=[str(c[0]) for c in CASES])
def test_predictor_matches_oracle(lengths, H, dh, b, d, rank):
    seed = sum(lengths) % 89
    x = synth.normal_bf16(sum(lengths), d, seed, 7)
    w1q, w2q, _ = synth.predictor_weights(d, rank, H * dh, 0.4, seed, 10)
    w1k, w2k, _ = synth.predictor_weights(d, rank, H * dh, 0.4, seed, 11)
    got, _ = run_predict(lengths, H, dh, b, x, w1q, w2q, w1k, w2k)
    want = oracle_predict(lengths, H, dh, b, x, w1q, w2q, w1k, w2k)
    err = assert_scores_close(got, want, "predicted scores")
    assert err < 1e-4


def test_many_short_sequences():
    """300 sequences: 64 x 64 tiles of block pairs span several sequences,
    whose cross pairs the block products must leave out."""
    rng = np.random.default_rng(41)
    lengths = [int(v) for v in rng.choice([0, 1, 63, 128, 129, 300], size=300)]
    H, dh, b, d, rank = 2, 32, 64, 64, 24
    x = synth.normal_bf16(sum(lengths), d, 41, 7)
    w1q, w2q, _ = synth.predictor_weights(d, rank, H * dh, 0.4, 41, 10)
    w1k, w2k, _ = synth.predictor_weights(d, rank, H * dh, 0.4, 41, 11)
    got, _ = run_predict(lengths, H, dh, b, x, w1q, w2q, w1k, w2k)
    want = oracle_predict(lengths, H, dh, b, x, w1q, w2q, w1k, w2k)
    assert_scores_close(got, want, "predicted scores, 300 sequences")
    # fp32 accuracy: one-token sequences give scores near 0, and a block pair's
    # 32-term dot products cancel (each product is exact to 2^-16, so the error
    # follows the size of the terms, not of the result); the error is measured
    # against the scale of the scores, and relatively (10x inside the 1e-2
    # bar) only for the scores that are not near 0
    scale = np.abs(want).max()
    assert np.abs(got - want).max() <= 1e-5 * scale
    big = np.abs(want) >= 1e-3 * scale
    assert (np.abs(got - want)[big] / np.abs(want[big])).max() < 1e-3


def test_weights_with_only_2_byte_alignment():
    """Weight pointers 2 bytes off a 16-byte boundary go through padded
    copies; the arithmetic is the same, so the scores are the same bits."""
    lengths, H, dh, b, d, rank = [640, 200], 2, 64, 64, 128, 48
    x = synth.normal_bf16(sum(lengths), d, 9, 7)
    w1q, w2q, _ = synth.predictor_weights(d, rank, H * dh, 0.4, 9, 10)
    w1k, w2k, _ = synth.predictor_weights(d, rank, H * dh, 0.4, 9, 11)
    aligned, _ = run_predict(lengths, H, dh, b, x, w1q, w2q, w1k, w2k)
    shifted, _ = run_predict(lengths, H, dh, b, x, w1q, w2q, w1k, w2k, misaligned=True)
    assert np.array_equal(aligned, shifted)
    assert_scores_close(shifted, oracle_predict(lengths, H, dh, b, x, w1q, w2q, w1k, w2k),
                        "predicted scores, misaligned weights")


def test_pruned_neurons_can_be_left_out():
    lengths, H, dh, b, d, rank = [700, 300], 2, 64, 64, 128, 64
    x = synth.normal_bf16(sum(lengths), d, 5, 7)
    w1q, w2q, lq = synth.predictor_weights(d, rank, H * dh, 0.4, 5, 10)
    w1k, w2k, lk = synth.predictor_weights(d, rank, H * dh, 0.4, 5, 11)
    full, _ = run_predict(lengths, H, dh, b, x, w1q, w2q, w1k, w2k)
    # the two predictors have different live sets: compact each to its own,
    # then pad to one rank per call with zero neurons (exact)
    q1, q2 = np.ascontiguousarray(w1q[:, lq]), np.ascontiguousarray(w2q[lq])
    k1, k2 = np.ascontiguousarray(w1k[:, lk]), np.ascontiguousarray(w2k[lk])
    r = max(len(lq), len(lk))
    def pad(w1, w2):
        a = np.zeros((d, r), np.uint16)
        c = np.zeros((r, H * dh), np.uint16)
        a[:, :w1.shape[1]] = w1
        c[:w2.shape[0]] = w2
        return a, c
    q1, q2 = pad(q1, q2)
    k1, k2 = pad(k1, k2)
    compact, _ = run_predict(lengths, H, dh, b, x, q1, q2, k1, k2)
    np.testing.assert_allclose(compact, full, rtol=1e-5, atol=1e-6 * np.abs(full).max())


def test_predictor_llama13b_32k_against_stored_oracle():
    key = "llama13b-32k"
    path = os.path.join(GOLDEN, f"{key}.json")
    if not os.path.exists(path):
        pytest.skip("no stored oracle values")
    with open(path) as f:
        g = json.load(f)["layers"][0]
    w = synth.WORKLOADS[key]
    x, _ = synth.projected_x(w.lengths[0], w.d, float(w.salient), w.seeds[0])
    y_out = synth.normal_bf16(w.total_L, w.d, w.seeds[0], 8)
    assert synth.digest(x, y_out) == g["digest_x"]
    w1q, w2q, _ = synth.predictor_weights(w.d, w.predictor_rank, w.H * w.dh, 0.4, w.seeds[0], 10)
    w1k, w2k, _ = synth.predictor_weights(w.d, w.predictor_rank, w.H * w.dh, 0.4, w.seeds[0], 11)
    assert synth.digest(w1q, w2q, w1k, w2k) == g["digest_pred"]
    got, cu = run_predict(list(w.lengths), w.H, w.dh, w.block, x, w1q, w2q, w1k, w2k)
    want = np.array([float(v) for v in g["pred_scores"]])
    assert_scores_close(got, want, "predicted scores llama13b-32k")
    ptheta = float(g["pred_theta"])
    mask_gpu = oracle.keep_mask(got.astype(np.float32), np.float32(ptheta))
    band = np.abs(want - ptheta) <= BAND * abs(ptheta)
    assert np.array_equal(mask_gpu[~band], oracle.keep_mask(want, ptheta)[~band])
    exact = np.array([float(v) for v in g["scores"]])
    rec = oracle.recall(mask_gpu, oracle.keep_mask(exact, float(g["theta"])))
    assert rec == pytest.approx(g["recall"], abs=2.0 / len(exact))


def test_grid_barrier_times_out_and_recovers():
    """One CTA of the persistent kernel withholds its arrival at the first
    grid barrier (test hook): every CTA's bounded wait runs out, the call
    reports LEMO_ERR_TIMEOUT and every CTA leaves (nothing hangs).  The next
    call, without the hook, gives the oracle's scores."""
    lengths, H, dh, b, d, rank = [1000, 300], 2, 64, 64, 128, 48
    x = synth.normal_bf16(sum(lengths), d, 13, 7)
    w1q, w2q, _ = synth.predictor_weights(d, rank, H * dh, 0.4, 13, 10)
    w1k, w2k, _ = synth.predictor_weights(d, rank, H * dh, 0.4, 13, 11)
    import torch
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    cu_d = torch.from_numpy(cu).cuda()
    shape = lemo.make_shape(cu_d, int(cu[-1]), max(lengths), H, dh, b)
    ws = torch.empty(lemo.lemo_predict_workspace_size(shape, d, rank), dtype=torch.uint8,
                     device="cuda")
    out = torch.zeros(32, dtype=torch.float32, device="cuda")
    try:
        lemo.lemo_set_test_hooks(-1, 50_000_000)
        lemo.lemo_set_predict_test_hook(0)
        lemo.lemo_predict_scores(shape, _dev(x), _dev(w1q), _dev(w2q), _dev(w1k), _dev(w2k),
                                 out, ws)
        assert lemo.lemo_get_error() == lemo.LEMO_ERR_TIMEOUT
    finally:
        lemo.lemo_set_predict_test_hook(-1)
        lemo.lemo_set_test_hooks(-1, 0)
    got, _ = run_predict(lengths, H, dh, b, x, w1q, w2q, w1k, w2k)
    assert_scores_close(got, oracle_predict(lengths, H, dh, b, x, w1q, w2q, w1k, w2k),
                        "predicted scores after a timed-out call")

"""GPU parity of the permutation-free attention over kept tokens.

The kernel computes scores and the running softmax in fp32, rounds the
probabilities to bf16 for the P V product (fp32 accumulation) and rounds the
output once.  Tolerance, per output element of head h (u = 2^-8):

    |got - O| <= u |O| + u max|V^h|

(rounding P moves each term p v by at most 2^-9 p |v| and the weights sum to
one; the output rounding adds 2^-9 |O|; fp32 score errors are far smaller).
In the in-place mode the exact sum x + O is rounded once more (another
2^-9 |x + O|); rows of eliminated tokens keep their bytes.
"""

import numpy as np
import pytest

import oracle
from contextual_token_sparsity_b200 import lemo, synth

pytestmark = pytest.mark.gpu
U = 2.0 ** -8
NAN_BF16 = 0x7FC0


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    torch.cuda.set_device(0)
    lemo.lemo_set_test_hooks(-1, 0)


def _dev16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


def _dev32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def kept_from_mask(lengths, b, mask):
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    idx, cu_kept, K = oracle.compact(np.asarray(mask, dtype=np.uint8), cu, b)
    return cu, np.asarray(idx[:K], dtype=np.int32), np.asarray(cu_kept, dtype=np.int32), int(K)


def random_kept(lengths, b, seed, p=0.5):
    nb = sum(-(-L // b) for L in lengths)
    mask = (np.random.default_rng(seed).random(nb) < p).astype(np.uint8)
    return kept_from_mask(lengths, b, mask)


def run_attention(lengths, H, dh, b, q, k, v, idx, cu_kept, K, x=None, scale=None,
                  poison_eliminated=False):
    """Returns (status, compact output bits or None, x bits or None)."""
    import torch
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    if poison_eliminated:  # eliminated rows of Q, K, V hold NaN: they must never matter
        keep = np.zeros(sum(lengths), dtype=bool)
        keep[idx] = True
        q, k, v = (np.where(keep[:, None], a, np.uint16(NAN_BF16)).astype(np.uint16)
                   for a in (q, k, v))
    cu_d = _dev32(cu)
    shape = lemo.make_shape(cu_d, int(cu[-1]), max(max(lengths), 1), H, dh, b)
    qd, kd, vd = _dev16(q), _dev16(k), _dev16(v)
    idx_d = _dev32(np.concatenate([idx, np.zeros(1, np.int32)]))
    cuk_d = _dev32(cu_kept)
    kt_d = _dev32(np.array([K]))
    ws = torch.empty(lemo.lemo_attention_workspace_size(len(lengths)), dtype=torch.uint8,
                     device="cuda")
    if x is None:
        o = torch.full((max(K, 1), H * dh), -1, dtype=torch.int16, device="cuda")
        lemo.lemo_attention_kept(shape, qd, kd, vd, idx_d, cuk_d, kt_d, ws, o=o, scale=scale)
        st = lemo.lemo_get_error()
        return st, o[:K].cpu().numpy().view(np.uint16), None
    xd = _dev16(x)
    lemo.lemo_attention_kept(shape, qd, kd, vd, idx_d, cuk_d, kt_d, ws, x=xd, scale=scale)
    st = lemo.lemo_get_error()
    return st, None, xd.cpu().numpy().view(np.uint16)


def vmax_per_head(v, H, dh):
    vf = np.abs(oracle.bf16_bits_to_f64(v)).reshape(-1, H, dh)
    return np.repeat(vf.max(axis=(0, 2)), dh)[None, :]


def check_compact(got_bits, want, v, H, dh):
    got = oracle.bf16_bits_to_f64(got_bits)
    tol = U * np.abs(want) + U * vmax_per_head(v, H, dh)
    err = np.abs(got - want)
    assert np.all(err <= tol), float((err / tol).max())


CASES = [
    ([300, 0, 517, 64, 1], 2, 64, 64, 0.6),     # varlen, empty and 1-token sequences
    ([1000], 3, 128, 64, 1.0),                   # everything kept: 8 key tiles
    ([1000, 777], 2, 128, 128, 0.5),             # block 128, short last blocks
    ([2049], 1, 128, 64, 0.5),
]


@pytest.mark.parametrize("lengths,H,dh,b,p", CASES, ids=[str(c[0]) + f"-dh{c[2]}-b{c[3]}"
                                                          for c in CASES])
def test_compact_output_matches_oracle(lengths, H, dh, b, p):
    seed = sum(lengths) % 97
    L = sum(lengths)
    q, k, v = (synth.normal_bf16(L, H * dh, seed, st) for st in (20, 21, 22))
    cu, idx, cu_kept, K = random_kept(lengths, b, seed, p)
    st, got, _ = run_attention(lengths, H, dh, b, q, k, v, idx, cu_kept, K)
    assert st == lemo.LEMO_OK, lemo.STATUS.get(st, st)
    want = oracle.attention_kept(q, k, v, idx, cu_kept, H, dh)
    check_compact(got, want, v, H, dh)


def test_many_short_sequences():
    """600 sequences with 0 to 5 kept blocks each (ragged last blocks,
    empty sequences): query-tile pairs and key tiles per sequence."""
    rng = np.random.default_rng(31)
    lengths = [int(v) for v in rng.choice([0, 1, 64, 65, 200, 300], size=600)]
    H, dh, b = 2, 64, 64
    L = sum(lengths)
    q, k, v = (synth.normal_bf16(L, H * dh, 31, st) for st in (20, 21, 22))
    cu, idx, cu_kept, K = random_kept(lengths, b, 31, 0.6)
    st, got, _ = run_attention(lengths, H, dh, b, q, k, v, idx, cu_kept, K)
    assert st == lemo.LEMO_OK, lemo.STATUS.get(st, st)
    check_compact(got, oracle.attention_kept(q, k, v, idx, cu_kept, H, dh), v, H, dh)


def test_in_place_residual_and_untouched_rows():
    lengths, H, dh, b = [700, 333], 2, 128, 64
    L = sum(lengths)
    q, k, v = (synth.normal_bf16(L, H * dh, 3, st) for st in (20, 21, 22))
    x = synth.normal_bf16(L, H * dh, 3, 23)
    cu, idx, cu_kept, K = random_kept(lengths, b, 4)
    st, _, xo = run_attention(lengths, H, dh, b, q, k, v, idx, cu_kept, K, x=x)
    assert st == lemo.LEMO_OK
    o = oracle.attention_kept(q, k, v, idx, cu_kept, H, dh)
    exact = oracle.attention_residual_exact(x, o, idx)
    others = np.setdiff1d(np.arange(L), idx)
    assert np.array_equal(xo[others], x[others])           # eliminated rows: same bytes
    got = oracle.bf16_bits_to_f64(xo[idx])
    tol = U * np.abs(exact[idx]) + U * vmax_per_head(v, H, dh)
    assert np.all(np.abs(got - exact[idx]) <= tol)


def test_eliminated_rows_are_never_read():
    lengths, H, dh, b = [517, 300], 2, 64, 64
    L = sum(lengths)
    q, k, v = (synth.normal_bf16(L, H * dh, 5, st) for st in (20, 21, 22))
    cu, idx, cu_kept, K = random_kept(lengths, b, 6)
    st, got, _ = run_attention(lengths, H, dh, b, q, k, v, idx, cu_kept, K,
                               poison_eliminated=True)
    assert st == lemo.LEMO_OK
    assert np.all(np.isfinite(oracle.bf16_bits_to_f64(got)))
    check_compact(got, oracle.attention_kept(q, k, v, idx, cu_kept, H, dh), v, H, dh)


def test_scale_and_large_logits():
    # large scores exercise the lazy rescaling of the running maximum
    lengths, H, dh, b = [900], 2, 128, 64
    q, k, v = (synth.normal_bf16(900, H * dh, 7, st) for st in (20, 21, 22))
    cu, idx, cu_kept, K = random_kept(lengths, b, 8, 0.8)
    for scale in (0.05, 1.0):
        st, got, _ = run_attention(lengths, H, dh, b, q, k, v, idx, cu_kept, K, scale=scale)
        assert st == lemo.LEMO_OK
        check_compact(got, oracle.attention_kept(q, k, v, idx, cu_kept, H, dh, scale=scale),
                      v, H, dh)


def test_nothing_kept_is_a_no_op():
    lengths, H, dh, b = [256, 128], 1, 64, 64
    q, k, v = (synth.normal_bf16(384, 64, 9, st) for st in (20, 21, 22))
    x = synth.normal_bf16(384, 64, 9, 23)
    cu, idx, cu_kept, K = kept_from_mask(lengths, b, np.zeros(6, np.uint8))
    assert K == 0
    st, _, xo = run_attention(lengths, H, dh, b, q, k, v, idx, cu_kept, K, x=x)
    assert st == lemo.LEMO_OK
    assert np.array_equal(xo, x)


def test_non_block_kept_set_is_reported():
    lengths, H, dh, b = [256], 1, 64, 64
    q, k, v = (synth.normal_bf16(256, 64, 10, st) for st in (20, 21, 22))
    idx = np.arange(0, 256, 2, dtype=np.int32)   # every other token: not whole blocks
    cu_kept = np.array([0, 128], dtype=np.int32)
    st, _, _ = run_attention(lengths, H, dh, b, q, k, v, idx, cu_kept, 128)
    assert st == lemo.LEMO_ERR_INVALID_ARG


def test_llama7b_16k_layer_sampled_rows():
    """Llama-2-7B layer shape (L = 16384, H = 32, dh = 128, b = 64) with the
    llama7b-16k layer-1 keep mask (50 %): sampled kept rows (at least one per
    128-row query tile) against the oracle."""
    import json
    import os
    L, H, dh, b = 16384, 32, 128, 64
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "llama7b-16k.json")
    with open(path) as f:
        g = json.load(f)["layers"][1]
    mask = oracle.keep_mask(np.array([float(s) for s in g["scores"]]), float(g["theta"]))
    q, k, v = (synth.normal_bf16(L, H * dh, 11, st) for st in (20, 21, 22))
    cu, idx, cu_kept, K = kept_from_mask([L], b, mask)
    st, got, _ = run_attention([L], H, dh, b, q, k, v, idx, cu_kept, K)
    assert st == lemo.LEMO_OK
    # one row in every 128-row query tile (at a seeded offset, so both query
    # tiles of a CTA and every key-tile boundary position are reached) plus
    # the tile edges and the last rows
    rng = np.random.default_rng(5)
    rows = sorted(set([0, 63, 64, 127, 128, 4095, K // 2, K - 129, K - 1] +
                      [t * 128 + int(rng.integers(0, 128)) for t in range(K // 128)]))
    rows = [r for r in rows if r < K]
    assert len(rows) >= 64
    want = oracle.attention_kept_rows(q, k, v, idx, cu_kept, H, dh, rows)
    check_compact(got[rows], want, v, H, dh)

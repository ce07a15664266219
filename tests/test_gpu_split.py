"""GPU checks of one long sequence split over key-tile shards.

lemo_score_blocks_shard computes the scores of one shard's key blocks with
the same tiles and arithmetic as lemo_score_blocks and writes 0 elsewhere,
so the shards' results summed are the unsharded scores bit for bit.  The
whole split flow (shard scores, sum, select / gather / scatter on token
shards) is run here rank after rank on one GPU, with the sum taken in place
of the all-reduce (no kernel waits on another), and compared with the
unsharded path.
"""

import numpy as np
import pytest

from contextual_token_sparsity_b200 import lemo, split, synth

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


def _bits(t):
    import torch
    return t.view(torch.int32).cpu().numpy()


@pytest.mark.parametrize("lengths,H,dh,b,world", [
    ([16384], 4, 128, 64, 2), ([16384], 4, 128, 64, 3), ([9000], 2, 64, 128, 4),
    ([3000, 0, 777, 5000], 2, 64, 64, 2), ([300], 2, 64, 64, 5)])
def test_shards_sum_to_unsharded_scores(lengths, H, dh, b, world):
    import torch
    from contextual_token_sparsity_b200.pipeline import Layer, to_device_bf16
    q, k, cu, _ = synth.qk_direct(lengths, H, dh, [0.1] * len(lengths), seed=sum(lengths) + world)
    qd, kd = to_device_bf16(q), to_device_bf16(k)
    layer = Layer(lengths, H, dh, b, d=8)
    full = layer.score(qd, kd).clone()
    assert lemo.lemo_get_error() == lemo.LEMO_OK
    nb = layer.total_blocks
    acc = torch.zeros_like(full)
    owners = np.zeros(nb, dtype=int)
    for r in range(world):
        part = torch.full_like(full, float("nan"))
        lemo.lemo_score_blocks_shard(layer.shape, qd, kd, 1.0, r, world, None, part, layer.ws)
        assert lemo.lemo_get_error() == lemo.LEMO_OK
        mine = np.concatenate([split.owned_blocks(L, b, r, world) for L in lengths])
        p = part[:nb].cpu().numpy()
        assert np.all(p[~mine] == 0.0)
        assert np.array_equal(_bits(part[:nb])[mine], _bits(full[:nb])[mine])
        owners += mine
        acc[:nb] += part[:nb]
    assert np.all(owners == 1)
    assert np.array_equal(_bits(acc[:nb]), _bits(full[:nb]))


@pytest.mark.parametrize("world", [2, 3])
def test_split_flow_matches_unsharded_layer(world):
    """Shard scores summed, then each rank's select / gather / scatter on its
    token shard: the kept rows in global order, the gathered rows and the
    updated residual equal the unsharded layer's."""
    import torch
    from contextual_token_sparsity_b200.pipeline import Layer, to_device_bf16
    L, H, dh, b, d = 16384, 4, 128, 64, 256
    q, k, cu, _ = synth.qk_direct([L], H, dh, [0.1], seed=77)
    x = synth.normal_bf16(L, d, 77, 7)
    y_out = synth.normal_bf16(L, d, 77, 8)
    qd, kd = to_device_bf16(q), to_device_bf16(k)
    ref = Layer([L], H, dh, b, d)
    s = ref.score(qd, kd).cpu().numpy()[: ref.total_blocks].astype(np.float64)
    theta = float(np.median(s))
    ref.select(theta)
    x_ref = to_device_bf16(x)
    y_ref = ref.gather(x_ref).clone()
    ref.scatter(x_ref, to_device_bf16(y_out))
    assert lemo.lemo_get_error() == lemo.LEMO_OK
    K = int(ref.kept_total.item())
    want_idx = ref.kept_idx[:K].cpu().numpy()

    ranks = [split.SplitLayer(L, H, dh, b, d, r, world) for r in range(world)]
    total = torch.zeros(ranks[0].nb, dtype=torch.float32, device="cuda")
    for sl in ranks:  # each rank's shard of the scores, then the sum (the all-reduce)
        lemo.lemo_score_blocks_shard(sl.shape, qd, kd, 1.0, sl.rank, world, None, sl.scores, sl.ws)
        total += sl.scores[: sl.nb]
    got_idx, counts = [], []
    for sl in ranks:
        sl.scores[: sl.nb].copy_(total)
        sl.select(theta)
        xs = to_device_bf16(x[sl.lo:sl.hi])
        ys = sl.gather(xs)
        Kr = int(sl.kept_total.item())
        off = sum(counts)
        # the sublayer output of this rank's kept rows, in the global kept order
        sl.scatter(xs, to_device_bf16(y_out[off:off + max(Kr, 1)]))
        assert lemo.lemo_get_error() == lemo.LEMO_OK
        idx = sl.kept_idx[:Kr].cpu().numpy() + sl.lo
        assert np.array_equal(ys[:Kr].view(torch.int16).cpu().numpy(),
                              y_ref[off:off + Kr].view(torch.int16).cpu().numpy())
        assert np.array_equal(xs.view(torch.int16).cpu().numpy(),
                              x_ref[sl.lo:sl.hi].view(torch.int16).cpu().numpy())
        got_idx.append(idx)
        counts.append(Kr)
    assert np.array_equal(np.concatenate(got_idx), want_idx)
    assert sum(counts) == K

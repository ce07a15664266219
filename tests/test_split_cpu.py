"""Host logic of one long sequence split over ranks (gloo, CPU).

The block scores are divided by key tiles (each rank scores the key blocks
of its own tiles and writes 0 elsewhere) and combined with one all-reduce
(sum); token movement is divided by token shards, and an all-gather of the
kept counts places each rank's kept rows in the global order.  Here the
per-rank scores come from the oracle restricted to the rank's key blocks (a
stand-in for the shard kernel, which the GPU tests check against the
unsharded kernel), so these tests check the partition and the combine logic:
the combined scores, the mask and the global kept ids equal the unsharded
oracle's, bit for bit.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASES = [(5000, 64), (3000, 128), (70, 64)]


def _worker(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from contextual_token_sparsity_b200 import split, synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        res = []
        for L, b in CASES:
            H, dh = 2, 16
            q, k, cu, _ = synth.qk_direct([L], H, dh, [0.1], seed=L + b)
            full = oracle.column_scores(oracle.score_blocks(q, k, cu, H, dh, b))
            # this rank's shard of the scoring, then the combine
            mine = split.owned_blocks(L, b, rank, world)
            part = torch.from_numpy(np.where(mine, full, 0.0))
            split.combine_scores(part, world)
            scores = part.numpy()
            theta = oracle.threshold_for_keep_ratio(full, 0.5)
            # token shard: select, compact, then place in the global order
            lo, hi = split.token_shard(L, b, rank, world)
            b_lo, b_hi = split.block_shard(L, b, rank, world)
            mask = oracle.keep_mask(scores[b_lo:b_hi], theta)
            idx, _, K = oracle.compact(mask, np.array([0, hi - lo]), b)
            offs = split.kept_offsets(torch.tensor([K], dtype=torch.int32), world)
            ids = [None] * world
            dist.all_gather_object(ids, (idx + lo).tolist())
            res.append((L, b, scores.tobytes() == full.tobytes(), mine.tolist(), offs.tolist(),
                        ids, int(K)))
        out.put((rank, res))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_split_sequence_matches_unsharded_oracle(world):
    import oracle
    from contextual_token_sparsity_b200 import split, synth
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = dict(out.get(timeout=10) for _ in range(world))
    for ci, (L, b) in enumerate(CASES):
        H, dh = 2, 16
        q, k, cu, _ = synth.qk_direct([L], H, dh, [0.1], seed=L + b)
        full = oracle.column_scores(oracle.score_blocks(q, k, cu, H, dh, b))
        theta = oracle.threshold_for_keep_ratio(full, 0.5)
        want_idx, _, want_K = oracle.compact(oracle.keep_mask(full, theta), cu, b)
        owners = np.zeros(len(full), dtype=int)
        for r in range(world):
            L_, b_, same, mine, offs, ids, K = got[r][ci]
            assert (L_, b_) == (L, b)
            assert same                                   # combined scores: bit for bit
            owners += np.array(mine, dtype=int)
            flat = [v for part in ids for v in part]
            assert flat == want_idx.tolist()              # global kept ids, in order
            assert offs[-1] == want_K
            assert offs[r + 1] - offs[r] == K == len(ids[r])
        assert np.all(owners == 1)                        # every key block scored once


def test_token_shards_and_owner_rule():
    from contextual_token_sparsity_b200 import split
    for L, b, world in [(16384, 64, 2), (16384, 64, 3), (1000, 128, 4), (64, 64, 3)]:
        rows = []
        for r in range(world):
            lo, hi = split.token_shard(L, b, r, world)
            assert lo % b == 0 and lo <= hi
            rows.append((lo, hi))
        assert rows[0][0] == 0 and rows[-1][1] == L
        assert all(rows[i][1] == rows[i + 1][0] for i in range(world - 1))
    # snake order: rounds alternate direction
    assert [split.key_tile_owner(kj, 3) for kj in range(9)] == [0, 1, 2, 2, 1, 0, 0, 1, 2]

"""One long sequence split over several GPUs (Jenga summary, section 6.4
"Scalability Analysis": the method scales without extra communication on its
data path).

The layer's work is divided two ways, one rank per GPU:

* block scoring by key tiles: key tile kj (256 tokens) belongs to rank
  ``key_tile_owner(kj, world)`` (snake order over rounds of ``world`` tiles);
  each rank runs ``lemo_score_blocks_shard`` for its tiles, which writes the
  complete scores of its key blocks and 0 elsewhere, and ONE all-reduce (sum)
  of the ``total_blocks`` floats gives every rank the unsharded scores, bit
  for bit (every score has exactly one non-zero contributor);
* token movement by token shards: rank r owns rows ``token_shard(...)`` of x
  (whole token blocks); it selects on its own blocks, gathers and scatters its
  own kept rows.  The per-rank kept counts are all-gathered and scanned so that
  each rank knows where its kept rows sit in the global kept order.

Q and K are replicated on every rank here (each rank's key tiles need every
later query tile); an all-gather of Q over NVLink would take their place when
each rank only holds its own rows.  Nothing else crosses GPUs: no TMA
multicast and no peer loads, only the two small NCCL collectives.
"""

from __future__ import annotations

import numpy as np

from . import lemo

KEY_TILE = 256  # key columns of one score tile of the scoring kernel


def key_tile_owner(kj: int, world: int) -> int:
    """Rank owning key tile kj: position kj % world of round kj // world,
    taken forwards in even rounds and backwards in odd ones."""
    rnd, pos = divmod(int(kj), int(world))
    return pos if rnd % 2 == 0 else world - 1 - pos


def owned_blocks(L: int, block: int, rank: int, world: int) -> np.ndarray:
    """Boolean mask of the token blocks of a sequence of L rows whose key
    tile belongs to `rank`."""
    nb = -(-int(L) // block)
    return np.array([key_tile_owner(m * block // KEY_TILE, world) == rank for m in range(nb)],
                    dtype=bool)


def block_shard(L: int, block: int, rank: int, world: int):
    """Token blocks [blo, bhi) of the token shard of `rank`: as even as
    possible (the last shards may be shorter or empty)."""
    nb = -(-int(L) // block)
    per = -(-nb // world)
    return min(rank * per, nb), min((rank + 1) * per, nb)


def token_shard(L: int, block: int, rank: int, world: int):
    """Rows [lo, hi) of the token shard of `rank` (whole blocks)."""
    blo, bhi = block_shard(L, block, rank, world)
    return min(blo * block, L), min(bhi * block, L)


def combine_scores(partial, world: int, group=None):
    """Sum the per-rank partial block scores in place (every rank ends with
    the full scores)."""
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return partial


def kept_offsets(kept_total, world: int, group=None):
    """Exclusive scan of the ranks' kept counts: element r is the position of
    rank r's first kept row in the global kept order, element `world` the
    global count.  ``kept_total`` is a one-element int32 tensor (device or
    host); the result is an int64 tensor on the same device."""
    import torch
    counts = kept_total.reshape(1).to(torch.int64)
    if world > 1:
        import torch.distributed as dist
        parts = [torch.empty_like(counts) for _ in range(world)]
        dist.all_gather(parts, counts, group=group)
        counts = torch.cat(parts)
    out = torch.zeros(world + 1, dtype=torch.int64, device=counts.device)
    out[1:] = torch.cumsum(counts, 0)
    return out


class SplitLayer:
    """One layer of one long sequence on rank `rank` of `world` GPUs: device
    buffers and the steps, in order (score -> combine -> select -> gather ->
    scatter).  ``x_shard`` passed to gather / scatter is this rank's rows of
    the residual; ``y_shard`` the sublayer output of this rank's kept rows, in
    their (compact) order."""

    def __init__(self, L: int, H: int, dh: int, block: int, d: int, rank: int, world: int,
                 pad_to: int = 128, device="cuda", group=None):
        import torch
        self.L, self.H, self.dh, self.block, self.d = int(L), H, dh, block, d
        self.rank, self.world, self.group, self.pad_to = rank, world, group, pad_to
        self.cu = torch.tensor([0, self.L], dtype=torch.int32, device=device)
        self.shape = lemo.make_shape(self.cu, self.L, self.L, H, dh, block)
        self.ws = torch.empty(lemo.lemo_workspace_size(self.shape), dtype=torch.uint8,
                              device=device)
        self.nb = -(-self.L // block)
        self.scores = torch.empty(max(self.nb, 1), dtype=torch.float32, device=device)
        self.lo, self.hi = token_shard(self.L, block, rank, world)
        self.b_lo, self.b_hi = block_shard(self.L, block, rank, world)
        Ls = self.hi - self.lo
        self.Ls = Ls
        self.cu_s = torch.tensor([0, Ls], dtype=torch.int32, device=device)
        self.shape_s = lemo.make_shape(self.cu_s, Ls, Ls, 1, 64, block)
        self.ws_s = torch.empty(max(lemo.lemo_workspace_size(self.shape_s), 256),
                                dtype=torch.uint8, device=device)
        nbs = max(self.b_hi - self.b_lo, 1)
        self.mask = torch.empty(nbs, dtype=torch.uint8, device=device)
        self.kept_idx = torch.empty(max(Ls, 1), dtype=torch.int32, device=device)
        self.cu_kept = torch.empty(2, dtype=torch.int32, device=device)
        self.kept_total = torch.empty(1, dtype=torch.int32, device=device)
        self.y = torch.empty((max(-(-Ls // pad_to) * pad_to, pad_to), d), dtype=torch.bfloat16,
                             device=device)

    def score(self, q, k, scale: float = 1.0, stream=None):
        """This rank's key tiles, then the all-reduce: full block scores."""
        lemo.lemo_score_blocks_shard(self.shape, q, k, scale, self.rank, self.world, None,
                                     self.scores, self.ws, stream)
        return combine_scores(self.scores[: self.nb], self.world, self.group)

    def select(self, theta: float, stream=None):
        """Threshold and compaction of this rank's token blocks (kept ids are
        rows of the shard)."""
        lemo.lemo_select(self.shape_s, self.scores[self.b_lo:], theta, self.mask, self.kept_idx,
                         self.cu_kept, self.kept_total, self.ws_s, stream)

    def gather(self, x_shard, stream=None):
        lemo.lemo_gather_pad(x_shard, self.kept_idx, self.kept_total, self.pad_to, self.y, stream)
        return self.y

    def scatter(self, x_shard, y_shard, stream=None):
        lemo.lemo_scatter_residual(x_shard, y_shard, self.kept_idx, self.kept_total, stream)

    def offsets(self):
        """Global position of this rank's first kept row, for every rank."""
        return kept_offsets(self.kept_total, self.world, self.group)

"""One layer of the path on a packed batch: device buffers and the four calls.

``Layer`` allocates (with torch, on the device) every buffer the C ABI
needs for a fixed batch layout and exposes the steps in order:

    layer.score(q, k)          block scores               (lemo_score_blocks)
    layer.select(theta)        mask + kept ids            (lemo_select)
    layer.gather(x)            y = x[kept] + zero tail     (lemo_gather_pad)
    layer.scatter(x, y_out)    x[kept] += y_out, in place  (lemo_scatter_residual)

No step copies anything to the host; K stays on the device.
"""

from __future__ import annotations

import numpy as np

from . import lemo


def _round_up(v: int, m: int) -> int:
    return (v + m - 1) // m * m


class Layer:
    def __init__(self, lengths, H: int, dh: int, block: int, d: int, pad_to: int = 128,
                 device="cuda", keep_block_max: bool = False):
        import torch
        self.torch = torch
        self.lengths = [int(v) for v in lengths]
        self.H, self.dh, self.block, self.d, self.pad_to = H, dh, block, d, pad_to
        self.total_L = int(sum(self.lengths))
        cu = np.zeros(len(self.lengths) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(self.lengths)
        self.cu_host = cu
        self.cu = torch.from_numpy(cu).to(device)
        self.shape = lemo.make_shape(self.cu, self.total_L, max(self.lengths), H, dh, block)
        ws = lemo.lemo_workspace_size(self.shape)
        if ws == 0:
            raise ValueError("invalid shape")
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
        self.nblocks = [-(-L // block) for L in self.lengths]
        self.total_blocks = int(sum(self.nblocks))
        self.block_scores = torch.empty(max(self.total_blocks, 1), dtype=torch.float32,
                                        device=device)
        self.block_max = (torch.full((max(lemo.lemo_block_max_elems(self.lengths, block), 1),),
                                     float("nan"), dtype=torch.float32, device=device)
                          if keep_block_max else None)
        self.mask = torch.empty(max(self.total_blocks, 1), dtype=torch.uint8, device=device)
        self.kept_idx = torch.empty(max(self.total_L, 1), dtype=torch.int32, device=device)
        self.cu_kept = torch.empty(len(self.lengths) + 1, dtype=torch.int32, device=device)
        self.kept_total = torch.empty(1, dtype=torch.int32, device=device)
        self.y_rows = max(_round_up(self.total_L, pad_to), pad_to)
        self.y = torch.empty((self.y_rows, d), dtype=torch.bfloat16, device=device)

    # -- the four steps ------------------------------------------------------
    def score(self, q, k, scale: float = 1.0, stream=None):
        lemo.lemo_score_blocks(self.shape, q, k, scale, self.block_max, self.block_scores,
                               self.ws, stream)
        return self.block_scores

    def select(self, theta: float, stream=None):
        lemo.lemo_select(self.shape, self.block_scores, theta, self.mask, self.kept_idx,
                         self.cu_kept, self.kept_total, self.ws, stream)

    def gather(self, x, stream=None):
        lemo.lemo_gather_pad(x, self.kept_idx, self.kept_total, self.pad_to, self.y, stream)
        return self.y

    def scatter(self, x, y_out, stream=None):
        lemo.lemo_scatter_residual(x, y_out, self.kept_idx, self.kept_total, stream)

    def step(self, q, k, theta: float, x, y_out, scale: float = 1.0, stream=None):
        """score -> select -> gather -> scatter on one stream."""
        self.score(q, k, scale, stream)
        self.select(theta, stream)
        self.gather(x, stream)
        self.scatter(x, y_out, stream)

    # -- helpers for checking results ----------------------------------------
    def block_max_list(self):
        """Per-sequence [N_b, N_b] numpy views of block_max (host copy)."""
        bm = self.block_max.cpu().numpy()
        out, off = [], 0
        for nb in self.nblocks:
            out.append(bm[off:off + nb * nb].reshape(nb, nb))
            off += nb * nb
        return out


def to_device_bf16(bits: np.ndarray, device="cuda"):
    """bf16 bit patterns (uint16 numpy) -> torch bfloat16 device tensor."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(
        torch.bfloat16)


def to_host_bits(t) -> np.ndarray:
    """torch bfloat16 tensor -> bf16 bit patterns (uint16 numpy)."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

"""Seeded synthetic inputs for the score -> select -> gather -> scatter path.

This module only draws inputs; it holds none of the method's arithmetic, so
both the CUDA path and the CPU oracle can be fed from it without sharing any
code with each other.  Every tensor is produced in float64/float32 by numpy's
PCG64 generator and rounded to bf16 here, so the oracle and the GPU see the
same bytes.

The shapes and value distributions follow the Llama-2 layer shapes used as
stand-ins for the pages' datasets and models (RedPajama / PG19 / Proof-Pile /
LongBench with OPT and Llama weights are not available): N(0, 1) queries and
keys with a salient subset of tokens whose per-head rows are stretched to 4x
their norm and turned onto one shared random direction per head, or queries
and keys projected from N(0, 1) embeddings with N(0, 1/d) weights.
"""

from __future__ import annotations

import dataclasses
import hashlib

import numpy as np

__all__ = [
    "to_bf16_bits",
    "bf16_bits_to_f32",
    "rng_for",
    "salient_rows",
    "qk_direct",
    "projected_x",
    "qk_projected",
    "normal_bf16",
    "predictor_weights",
    "mlp_activations",
    "Workload",
    "WORKLOADS",
    "make_workload",
    "digest",
]


def to_bf16_bits(a) -> np.ndarray:
    """float -> bf16 bit patterns: first to float32 (numpy rounding), then
    the float32 pattern is rounded to its upper 16 bits, ties to even."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32)
    r = (u >> 16) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u  # cannot wrap for finite values (only NaN patterns are that large)
    r >>= np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def rng_for(seed: int, stream: int) -> np.random.Generator:
    """Independent, reproducible stream ``stream`` of seed ``seed``."""
    return np.random.default_rng([int(seed), int(stream)])


def salient_rows(rng: np.random.Generator, L: int, frac: float) -> np.ndarray:
    """round(frac * L) distinct token ids, sorted."""
    n = int(np.floor(frac * L + 0.5))
    return np.sort(rng.choice(L, size=n, replace=False)) if n else np.zeros(0, np.int64)


def qk_direct(lengths, H: int, dh: int, salient_fracs, seed: int):
    """Queries and keys drawn directly (Llama-2 layer shapes).

    Q, K ~ N(0, 1) of shape [total_L, H, dh].  In each sequence a salient
    subset of round(f * L) tokens is drawn; for those tokens every head's row
    of Q and of K is replaced by 4 * ||row|| * u_h, where u_h is one random
    unit vector per head shared by all salient tokens (of Q and of K).
    Returns (q_bits, k_bits, cu_seqlens int32, salient global ids).
    """
    lengths = [int(L) for L in lengths]
    total = sum(lengths)
    rq, rk, rs = rng_for(seed, 1), rng_for(seed, 2), rng_for(seed, 3)
    q = rq.standard_normal((total, H, dh), dtype=np.float32)
    k = rk.standard_normal((total, H, dh), dtype=np.float32)
    u = rs.standard_normal((H, dh))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    u = u.astype(np.float32)
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    sal = []
    for s, L in enumerate(lengths):
        ids = cu[s] + salient_rows(rs, L, float(salient_fracs[s]))
        sal.append(ids)
        for t in (q, k):
            nrm = np.linalg.norm(t[ids], axis=2, keepdims=True)  # [n, H, 1]
            t[ids] = 4.0 * nrm * u[None, :, :]
    sal = np.concatenate(sal) if sal else np.zeros(0, np.int64)
    return (to_bf16_bits(q).reshape(total, H * dh), to_bf16_bits(k).reshape(total, H * dh),
            cu, sal)


def projected_x(L: int, d: int, salient_frac: float, seed: int):
    """Embeddings X ~ N(0, 1) [L, d] with round(frac * L) salient rows scaled
    by 4, as bf16 bits; returns (x_bits, salient ids)."""
    rx = rng_for(seed, 4)
    x = rx.standard_normal((L, d), dtype=np.float32)
    sal = salient_rows(rx, L, salient_frac)
    x[sal] *= 4.0
    return to_bf16_bits(x), sal


def qk_projected(L: int, d: int, H: int, dh: int, salient_frac: float, seed: int,
                 chunk: int = 4096):
    """Embeddings X ~ N(0, 1) [L, d] with a salient subset scaled by 4, and
    Q = bf16(X Wq), K = bf16(X Wk) with Wq, Wk ~ N(0, 1/d) [d, H*dh].

    X and the weights are rounded to bf16 first; the projections are computed
    in float64 from those bf16 values (row chunks of ``chunk``) and rounded.
    Returns (x_bits [L, d], q_bits [L, H*dh], k_bits [L, H*dh], salient ids).
    """
    x_bits, sal = projected_x(L, d, salient_frac, seed)
    rw = rng_for(seed, 5)
    std = 1.0 / np.sqrt(d)
    wq = bf16_bits_to_f32(to_bf16_bits(rw.standard_normal((d, H * dh)) * std)).astype(np.float64)
    wk = bf16_bits_to_f32(to_bf16_bits(rw.standard_normal((d, H * dh)) * std)).astype(np.float64)
    q_bits = np.empty((L, H * dh), dtype=np.uint16)
    k_bits = np.empty((L, H * dh), dtype=np.uint16)
    for r0 in range(0, L, chunk):
        xc = bf16_bits_to_f32(x_bits[r0:r0 + chunk]).astype(np.float64)
        q_bits[r0:r0 + chunk] = to_bf16_bits(xc @ wq)
        k_bits[r0:r0 + chunk] = to_bf16_bits(xc @ wk)
    return x_bits, q_bits, k_bits, sal


def normal_bf16(rows: int, cols: int, seed: int, stream: int) -> np.ndarray:
    """bf16 bits of an N(0, 1) [rows, cols] matrix."""
    return to_bf16_bits(rng_for(seed, stream).standard_normal((rows, cols), dtype=np.float32))


def predictor_weights(d: int, rank: int, out: int, zero_frac: float, seed: int, stream: int):
    """Two-matrix low-rank ReLU predictor W1 [d, rank] ~ N(0, 1/d),
    W2 [rank, out] ~ N(0, 1/rank), with floor(zero_frac * rank) hidden
    neurons zeroed (their W1 column and W2 row), as an elastic-size pruning
    would leave them.  Returns (w1_bits, w2_bits, live neuron ids)."""
    r = rng_for(seed, stream)
    w1 = r.standard_normal((d, rank)) / np.sqrt(d)
    w2 = r.standard_normal((rank, out)) / np.sqrt(rank)
    dead = np.sort(r.choice(rank, size=int(np.floor(zero_frac * rank)), replace=False))
    w1[:, dead] = 0.0
    w2[dead, :] = 0.0
    live = np.setdiff1d(np.arange(rank), dead)
    return to_bf16_bits(w1), to_bf16_bits(w2), live


def mlp_activations(L: int, d_ff: int, salient_frac: float, seed: int, gated: bool = True):
    """MLP intermediate activations at a layer's shape: gate, up ~ N(0, 1)
    [L, d_ff] (SiLU-gated MLP) or ReLU outputs relu(N(0, 1)) (ReLU MLP), with
    round(frac * L) salient token rows scaled by 4.  Returns bf16 bits:
    (gate, up) or (act,)."""
    r = rng_for(seed, 12)
    sal = salient_rows(r, L, salient_frac)
    if gated:
        g = r.standard_normal((L, d_ff), dtype=np.float32)
        u = r.standard_normal((L, d_ff), dtype=np.float32)
        g[sal] *= 4.0
        u[sal] *= 4.0
        return to_bf16_bits(g), to_bf16_bits(u)
    a = np.maximum(r.standard_normal((L, d_ff), dtype=np.float32), 0.0)
    a[sal] *= 4.0
    return (to_bf16_bits(a),)


def lm_head_inputs(T: int, d: int, V: int, seed: int, logit_std: float = 2.0,
                   ignore_frac: float = 0.0, ignore_index: int = -100):
    """Inputs of the lm-head loss: final hidden states h ~ N(0, 1) [T, d],
    lm-head weight W ~ N(0, logit_std^2 / d) [V, d] (logits of standard
    deviation about logit_std), uniform next-token targets in [0, V) with a
    seeded fraction set to ``ignore_index``.  Returns (h bits, W bits, int32
    targets)."""
    r = rng_for(seed, 13)
    h = to_bf16_bits(r.standard_normal((T, d), dtype=np.float32))
    w = r.standard_normal((V, d), dtype=np.float32)
    w *= np.float32(logit_std / np.sqrt(d))
    y = r.integers(0, V, size=T).astype(np.int32)
    if ignore_frac > 0:
        y[r.random(T) < ignore_frac] = ignore_index
    return h, to_bf16_bits(w), y


# Segmented lm-head loss at the Llama-2-7B head (d = 4096, V = 32000) over
# the 16384 tokens of one long sequence, 16 segments of 1024 tokens.
LM_HEAD_WORKLOADS = {
    "lmhead-llama7b-16k": dict(T=16384, d=4096, V=32000, seg_rows=1024, seed=0),
}


@dataclasses.dataclass
class Workload:
    """One configuration of the path: shapes, seeds and keep ratios."""
    name: str
    lengths: tuple
    d: int
    H: int
    dh: int
    block: int
    keep: tuple            # keep ratio per layer
    seeds: tuple           # one seed per layer
    kind: str              # "direct" or "projected"
    salient: object = 0.1  # fraction, or "uniform-5-20" per sequence
    predictor_rank: int = 0

    @property
    def total_L(self) -> int:
        return int(sum(self.lengths))

    @property
    def layers(self) -> int:
        return len(self.keep)


WORKLOADS = {
    "small-1k": Workload("single layer L=1024 d=512 H=8 dh=64 b=64", (1024,), 512, 8, 64, 64,
                   (0.5,), (0,), "projected"),
    "llama7b-8k": Workload("llama2-7b layer L=8192 d=4096 H=32 dh=128 b=64 keep 50%", (8192,),
                           4096, 32, 128, 64, (0.5,), (0,), "direct"),
    "llama7b-16k": Workload("llama2-7b layers L=16384 d=4096 H=32 dh=128 b=64 keep 30/50/70%",
                   (16384,), 4096, 32, 128, 64, (0.3, 0.5, 0.7), (0, 1, 2), "direct"),
    "varlen-10k": Workload("varlen L={4096,3072,2048,1024} d=4096 H=32 dh=128 b=64 keep 50%",
                   (4096, 3072, 2048, 1024), 4096, 32, 128, 64, (0.5,), (0,), "direct",
                   salient="uniform-5-20"),
    "llama13b-32k": Workload("llama2-13b layer L=32768 d=5120 H=40 dh=128 b=128 keep 50% "
                             "+ predictor",
                   (32768,), 5120, 40, 128, 128, (0.5,), (0,), "projected",
                   predictor_rank=256),
}


def make_workload(key: str, layer: int = 0, with_x: bool = True):
    """Generate one layer of a configuration.

    Returns a dict with bf16 bit arrays ``q``, ``k`` ([total_L, H*dh]),
    ``cu_seqlens`` (int32), ``x`` (residual stream [total_L, d]), ``y_out``
    (stand-in sublayer output [total_L, d], N(0, 1)), and for the predictor
    configuration ``w1q, w2q, w1k, w2k``.
    """
    w = WORKLOADS[key]
    seed = int(w.seeds[layer])
    out = {"workload": w, "layer": layer}
    if w.kind == "direct":
        if w.salient == "uniform-5-20":
            fr = rng_for(seed, 6).uniform(0.05, 0.20, size=len(w.lengths))
        else:
            fr = [float(w.salient)] * len(w.lengths)
        q, k, cu, sal = qk_direct(w.lengths, w.H, w.dh, fr, seed)
        out.update(q=q, k=k, cu_seqlens=cu, salient=sal, salient_fracs=np.asarray(fr))
        if with_x:
            out["x"] = normal_bf16(w.total_L, w.d, seed, 7)
    else:
        assert len(w.lengths) == 1
        x, q, k, sal = qk_projected(w.lengths[0], w.d, w.H, w.dh, float(w.salient), seed)
        cu = np.array([0, w.lengths[0]], dtype=np.int32)
        out.update(q=q, k=k, cu_seqlens=cu, salient=sal, x=x)
        if w.predictor_rank:
            w1q, w2q, liveq = predictor_weights(w.d, w.predictor_rank, w.H * w.dh, 0.4, seed, 10)
            w1k, w2k, livek = predictor_weights(w.d, w.predictor_rank, w.H * w.dh, 0.4, seed, 11)
            out.update(w1q=w1q, w2q=w2q, w1k=w1k, w2k=w2k, live_q=liveq, live_k=livek)
    if with_x:
        out["y_out"] = normal_bf16(w.total_L, w.d, seed, 8)
    return out


def digest(*arrays) -> str:
    """sha256 over the raw bytes of the given arrays (input fingerprints)."""
    h = hashlib.sha256()
    for a in arrays:
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()

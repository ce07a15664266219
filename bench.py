"""Throughput of the contextual-token-sparsity hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lemo|reference]
                    [--workload llama7b-16k]

One step is one pass of the whole path - block scores, threshold, compaction,
gather, scatter with residual add - over every layer of the workload (default:
three Llama-2-7B layers at L = 16384, H = 32, dh = 128, b = 64, d = 4096 with
keep ratios 30/50/70 %).  The metric is tokens per second per layer: layers x
tokens / step time.  Inputs are seeded synthetic data already resident in HBM
when the timed region starts; each step streams ~1 GB of Q/K/residual rows,
far more than the 126 MB L2, so L2 is not flushed between steps.

Prints ONE JSON line (rank 0).  With --gpus N > 1 (under torchrun) every rank
runs its own copy of the workload (independent layers, no collective on the
data path: weak scaling); the step time is the maximum over ranks.

``--impl reference`` times the CPU oracle (float64 numpy, the repository's
correctness reference) on a bounded sample of the same workload, as the
reference arm.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "tokens/sec per layer (score+select+gather+scatter) and % of roofline"
UNIT = "tokens/s"
PAD_TO = 128
LAUNCHES_PER_LAYER = 7  # plan+score+colsum, plan+select, gather, scatter
SCORE_SOURCES = ["score.cuh", "common.cuh", "tile_plan.h"]


# ----------------------------------------------------------------------------
# ranks
# ----------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Maximum of a float over all ranks (identity for one rank)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    return units_per_rank * world / max_seconds


def barrier(world: int, local: int, cuda: bool = True):
    if world > 1:
        import torch.distributed as dist
        if cuda:
            dist.barrier(device_ids=[local])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------
# algorithmic work of the path (per layer)
# ----------------------------------------------------------------------------

def score_flops(lengths, H, dh) -> float:
    """2 flops per multiply-add over the causal pairs i > j of every sequence."""
    return float(sum(H * dh * L * (L - 1) for L in lengths))


def move_bytes(K: int, d: int, pad_to: int = PAD_TO):
    K_pad = -(-K // pad_to) * pad_to
    gather = 4 * K * d + 2 * (K_pad - K) * d + 4 * K
    scatter = 6 * K * d + 4 * K
    return gather, scatter


def select_bytes(total_L: int, nblocks: int, K: int, batch: int) -> int:
    return 4 * nblocks + nblocks + 4 * K + 4 * (batch + 1) * 2 + 4


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def score_source_digest() -> str:
    h = hashlib.sha256()
    for name in SCORE_SOURCES:
        with open(os.path.join(ROOT, "contextual_token_sparsity_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per scorer launch from the committed ncu record
    (profiles/score_tiles_traffic.json), if it was taken on this workload and
    on the current scorer source (else None)."""
    path = os.path.join(ROOT, "profiles", "score_tiles_traffic.json")
    if not os.path.exists(path):
        return None
    try:
        with open(path) as f:
            rec = json.load(f)
        if rec.get("workload") != workload or rec.get("source_digest") != score_source_digest():
            return None
        return int(rec["dram_bytes_per_launch"])
    except (KeyError, ValueError, TypeError):
        return None


def headline_config(key: str, w, kept, thetas, theta_src: str, world: int) -> dict:
    """The `config` object of a headline-workload line; both arms print the
    same one."""
    nl = w.layers
    return {"workload": f"{key}: {w.name}", "layers": nl,
            "seq_lens": list(w.lengths), "heads": w.H, "head_dim": w.dh,
            "block": w.block, "d": w.d, "keep": list(w.keep), "kept_tokens": list(kept),
            "thresholds": thetas, "threshold_source": theta_src, "pad_to": PAD_TO,
            "l2": "not flushed; each step streams "
                  f"{(nl * (2 * w.total_L * w.H * w.dh * 2) + 3 * w.total_L * w.d * 2) / 1e9:.2f}"
                  " GB of Q/K/residual rows (> 126 MB L2)",
            "parallelism": f"{world} independent replica(s), no collective"}


def thresholds(key: str, layers: int):
    """Per-layer thresholds stored by the oracle-only golden script."""
    path = os.path.join(ROOT, "tests", "golden", f"{key}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        g = json.load(f)
    return [float(g["layers"][l]["theta"]) for l in range(layers)]


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------

class ClockSampler:
    """Clock, power and throttle-reason samples of one GPU while a timed
    region runs: NVML polled from a thread every 10 ms (read-only queries),
    or nvidia-smi every 100 ms where NVML cannot be loaded."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    PERIOD_S = 0.01

    def __init__(self, index):
        self.index = index  # a GPU UUID ("GPU-...") or an index
        self.proc = None
        self.nv = None
        self.rows = []
        self.path = os.path.join("/tmp", f"lemo_clocks_{os.getpid()}_{index}.csv")

    def start(self):
        if self._start_nvml():
            return
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def _start_nvml(self) -> bool:
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
        except Exception:
            return False
        try:
            idx = str(self.index)
            h = (nv.nvmlDeviceGetHandleByUUID(idx) if idx.startswith("GPU-")
                 else nv.nvmlDeviceGetHandleByIndex(int(idx)))
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:
            nv.nvmlShutdown()
            return False
        self.nv, self.h = nv, h
        self.bits = (nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                     nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap)
        self.halt = threading.Event()
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()
        return True

    def _poll(self):
        nv, h = self.nv, self.h
        while not self.halt.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.rows.append((sm, self.max_mhz, pw,
                                  [self.REASONS[i] for i, b in enumerate(self.bits) if rs & b]))
            except Exception:
                pass
            self.halt.wait(self.PERIOD_S)

    def stop(self):
        if self.nv is not None:
            self.halt.set()
            self.thread.join(timeout=5)
            self.nv.nvmlShutdown()
            return self.summary(self.rows, "nvml")
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 8:
                    rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        return self.summary([self.parse_smi(r) for r in rows], "nvidia-smi")

    @classmethod
    def parse_smi(cls, r):
        """One nvidia-smi CSV row -> (sm MHz, max MHz, power W, active reasons)."""
        def num(v):
            try:
                return float(v)
            except ValueError:
                return float("nan")
        return (num(r[0]), num(r[1]), num(r[2]),
                [cls.REASONS[i] for i in range(4) if r[4 + i].lower() == "active"])

    @staticmethod
    def summary(rows, source):
        if not rows:
            return None
        sm = [r[0] for r in rows if not math.isnan(r[0])]
        mx = [r[1] for r in rows if not math.isnan(r[1])]
        pw = [r[2] for r in rows if not math.isnan(r[2])]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "samples": len(rows),
                "power_w_median": statistics.median(pw) if pw else None,
                "power_w_max": max(pw) if pw else None,
                "reasons": sorted({x for r in rows for x in r[3]}),
                "source": source}


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------

def run_lemo(args):
    import torch

    from contextual_token_sparsity_b200 import lemo, synth
    from contextual_token_sparsity_b200.pipeline import Layer, to_device_bf16

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    lemo.load()

    w = synth.WORKLOADS[args.workload]
    nl = w.layers
    thetas = thresholds(args.workload, nl)
    theta_src = "oracle scores (tests/golden)"

    # inputs: per layer Q, K and sublayer output; one residual stream x
    host = [synth.make_workload(args.workload, l, with_x=True) for l in range(nl)]
    layers = [Layer(w.lengths, w.H, w.dh, w.block, w.d, pad_to=PAD_TO, device=dev)
              for _ in range(nl)]
    q = [to_device_bf16(h["q"], dev) for h in host]
    k = [to_device_bf16(h["k"], dev) for h in host]
    y_out = [to_device_bf16(h["y_out"], dev) for h in host]
    x0 = to_device_bf16(host[0]["x"], dev)
    x = x0.clone()
    if thetas is None:  # no stored oracle thresholds: derive from this GPU's scores
        thetas = []
        for l in range(nl):
            s = layers[l].score(q[l], k[l]).cpu().numpy()[: layers[l].total_blocks]
            srt = np.sort(s.astype(np.float64))[::-1]
            kk = int(math.floor(w.keep[l] * srt.size + 0.5))
            thetas.append(float(0.5 * (srt[kk - 1] + srt[kk])))
        theta_src = "keep ratio on GPU scores"
    stream = torch.cuda.current_stream(dev)

    comp = ("score", "select", "gather", "scatter")

    def step(evs=None):
        for l in range(nl):
            L_ = layers[l]
            if evs is not None:
                evs[l][0].record(stream)
            L_.score(q[l], k[l])
            if evs is not None:
                evs[l][1].record(stream)
            L_.select(thetas[l])
            if evs is not None:
                evs[l][2].record(stream)
            L_.gather(x)
            if evs is not None:
                evs[l][3].record(stream)
            L_.scatter(x, y_out[l])
            if evs is not None:
                evs[l][4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = lemo.lemo_get_error()
    if st != lemo.LEMO_OK:
        raise RuntimeError(f"device error during warm-up: {lemo.STATUS.get(st, st)}")
    kept = [int(L_.kept_total.item()) for L_ in layers]

    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(local)
    clocks = ClockSampler(gpu_id)
    clocks.start()
    time.sleep(0.3)
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(nl)]
          for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(world, local)
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        step(ev[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world, local)
    elapsed_s = t_start.elapsed_time(t_end) / 1e3
    clk = clocks.stop()
    st = lemo.lemo_get_error()
    if st != lemo.LEMO_OK:
        raise RuntimeError(f"device error in timed region: {lemo.STATUS.get(st, st)}")
    max_s = max_over_ranks(elapsed_s, world, dev)

    comp_ms = {c: [] for c in comp}
    for i in range(args.steps):
        for l in range(nl):
            for ci, c in enumerate(comp):
                comp_ms[c].append(ev[i][l][ci].elapsed_time(ev[i][l][ci + 1]))
    avg_us = {c: 1e3 * statistics.fmean(v) for c, v in comp_ms.items()}

    tokens_per_step = nl * w.total_L
    value = whole_job_rate(tokens_per_step, world, max_s / args.steps)

    # roofline of the dominant kernel (the scorer: dense contraction -> tensor)
    peaks = load_peaks()
    F = score_flops(w.lengths, w.H, w.dh)
    score_s = avg_us["score"] / 1e6
    long_region = elapsed_s > 2.0
    peak_tf = peaks["bf16_tflops_sustained"] if long_region else peaks["bf16_tflops"]
    achieved_tf = F / score_s / 1e12
    traffic = profiled_traffic(args.workload)
    roofline = {"bound": "tensor", "kernel": "score_tiles_kernel (+plan, column sum)",
                "achieved": round(achieved_tf, 1), "peak": peak_tf, "unit": "TFLOP/s",
                "frac": round(achieved_tf / peak_tf, 4), "traffic": traffic,
                "frac_of_sustained_peak": round(achieved_tf / peaks["bf16_tflops_sustained"], 4),
                "peak_source": f"{peaks['source']} bf16 "
                               f"{'sustained' if long_region else 'burst'} cuBLAS GEMM",
                "algorithmic_flops_per_launch": F}
    # whole-path roofline: scorer at the tensor peak + movement at HBM bandwidth
    bw = peaks["hbm_gbs"] * 1e9
    movement = []
    t_roof = 0.0
    for l in range(nl):
        g_b, s_b = move_bytes(kept[l], w.d)
        sel_b = select_bytes(w.total_L, layers[l].total_blocks, kept[l], len(w.lengths))
        t_roof += F / (peak_tf * 1e12) + (g_b + s_b + sel_b) / bw
        movement.append({"K": kept[l], "gather_bytes": g_b, "scatter_bytes": s_b})
    gather_gbs = statistics.fmean(
        move_bytes(kept[l], w.d)[0] for l in range(nl)) / (avg_us["gather"] / 1e6) / 1e9
    scatter_gbs = statistics.fmean(
        move_bytes(kept[l], w.d)[1] for l in range(nl)) / (avg_us["scatter"] / 1e6) / 1e9
    step_s = max_s / args.steps

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_s * 1e3, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": headline_config(args.workload, w, kept, thetas, theta_src, world),
        "roofline": roofline,
        "path_roofline": {"frac": round(t_roof / step_s, 4),
                          "roofline_ms_per_step": round(t_roof * 1e3, 4),
                          "model": "scorer flops at the bf16 peak + select/gather/scatter "
                                   "bytes at the HBM copy bandwidth"},
        "kernels_us": {c: round(v, 2) for c, v in avg_us.items()},
        "movement": {"gather_gbs": round(gather_gbs, 1), "scatter_gbs": round(scatter_gbs, 1),
                     "hbm_peak_gbs": peaks["hbm_gbs"],
                     "gather_frac": round(gather_gbs / peaks["hbm_gbs"], 4),
                     "scatter_frac": round(scatter_gbs / peaks["hbm_gbs"], 4)},
        "gpu_launches": LAUNCHES_PER_LAYER * nl * args.steps,
        "clocks": clk,
    }

    # the naive token movement beside the fused one (outside the timed region)
    fused_us = [1e3 * statistics.fmean(ev[i][l][2].elapsed_time(ev[i][l][4])
                                       for i in range(args.steps)) for l in range(nl)]
    out["naive_movement"] = naive_movement(x, y_out, layers, kept, fused_us)

    # end to end through the C ABI with host buffers: H2D of each layer's
    # Q/K/sublayer output and of the residual, the path, D2H of the residual
    # and of the block scores, every step.
    if not args.no_e2e:
        out["e2e"] = run_e2e(args, host, layers, thetas, dev, world, local, tokens_per_step)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.workload, budget_s=args.cpu_seconds)

    if world == 1 and not args.no_extensions:
        del q, k, y_out, x0, x, layers
        out["extensions"] = run_extensions(args)

    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


EXTENSIONS = ("predict-llama13b-32k", "lmhead-llama7b-16k", "attn-llama7b-16k", "mlp-llama7b-16k")


def run_extensions(args):
    """Each extension workload, briefly, in the same run (one GPU): the
    summary of its own line - throughput, time per step, the roofline of its
    dominant kernel, per-kernel times and the clocks - so that every row is
    measured by the default benchmark run.  The full line (with e2e and the
    CPU oracle) comes from `bench.py --workload W`."""
    import copy

    import torch
    global _COLLECT
    res = {}
    for wl in EXTENSIONS:
        sub = copy.copy(args)
        sub.workload = wl
        sub.steps = max(3, min(args.steps, 10))
        sub.warmup = 3
        sub.no_e2e = True
        sub.no_cpu_baseline = True
        _COLLECT = []
        try:
            {"lmhead-llama7b-16k": run_segloss, "attn-llama7b-16k": run_attention,
             "predict-llama13b-32k": run_predict, "mlp-llama7b-16k": run_mlp}[wl](sub)
            o = _COLLECT[-1]
            r = o.get("roofline", {})
            res[wl] = {"metric": o["metric"], "value": o["value"], "unit": o["unit"],
                       "steps": o["steps"], "ms_per_step": o["ms_per_step"],
                       "roofline": {k_: r.get(k_) for k_ in ("bound", "kernel", "achieved", "peak",
                                                             "unit", "frac")},
                       "kernels_us": o.get("kernels_us"), "clocks": o.get("clocks")}
        except Exception as e:  # noqa: BLE001 - reported, not hidden
            res[wl] = {"error": f"{type(e).__name__}: {e}"}
        finally:
            _COLLECT = None
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
    return res


def naive_movement(x, y_out, layers, kept, fused_us, reps: int = 10):
    """Time the naive token movement that permutation-free movement replaces
    (Jenga summary, section 4.2.3, and Fig. 18 of section 6.2) beside the
    fused gather + scatter of each layer, outside the timed region:

        eliminate      xk = x.index_select(0, kept)          (compact copy of the kept rows)
        re-permute     o = zeros_like(x); o.index_copy_(0, kept, y[:K])   (zero-padded,
                       original token order)
        residual add   x.add_(o)                              (over all L rows)

    (PyTorch ops, a comparator only; the sublayer between them is not
    timed).  Also checks on a copy of x that both give the same bits."""
    import torch
    stream = torch.cuda.current_stream(x.device)
    res = {"naive_us_per_layer": [], "fused_us_per_layer": [round(v, 2) for v in fused_us],
           "naive_ops": "torch index_select; zeros_like + index_copy_; full-length add_",
           "fused_ops": "lemo_gather_pad + lemo_scatter_residual (kept rows only)",
           "pages": "10x to over 50x, growing with sequence length (Jenga Fig. 18; hardware "
                    "and naive implementation not stated)", "matches_fused": True}
    for l, L_ in enumerate(layers):
        K = kept[l]
        idx = L_.kept_idx[:K].long()
        yk = y_out[l][:K]
        xw = x.clone()

        def naive():
            xk = xw.index_select(0, idx)
            o = torch.zeros_like(xw)
            o.index_copy_(0, idx, yk)
            xw.add_(o)
            return xk

        for _ in range(2):
            naive()
        ts = []
        for _ in range(reps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            naive()
            b.record(stream)
            b.synchronize()
            ts.append(1e3 * a.elapsed_time(b))
        res["naive_us_per_layer"].append(round(statistics.median(ts), 2))
        # same bits: the naive path and the fused path on one copy of x each
        xa, xb = x.clone(), x.clone()
        torch.cuda.synchronize()
        xk = xa.index_select(0, idx)
        o = torch.zeros_like(xa)
        o.index_copy_(0, idx, yk)
        xa.add_(o)
        g = L_.gather(xb)
        L_.scatter(xb, y_out[l])
        torch.cuda.synchronize()
        same = bool(torch.equal(xa.view(torch.int16), xb.view(torch.int16))) and \
            bool(torch.equal(xk.view(torch.int16), g[:K].view(torch.int16)))
        res["matches_fused"] = res["matches_fused"] and same
    res["speedup_per_layer"] = [round(n / f, 2) for n, f in
                                zip(res["naive_us_per_layer"], res["fused_us_per_layer"])]
    return res


def run_e2e(args, host, layers, thetas, dev, world, local, tokens_per_step):
    import torch
    nl = len(layers)
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()  # noqa
    hq = [pin(h["q"]) for h in host]
    hk = [pin(h["k"]) for h in host]
    hy = [pin(h["y_out"]) for h in host]
    hx = pin(host[0]["x"])
    hx_out = torch.empty_like(hx).pin_memory()
    hs_out = [torch.empty(L_.block_scores.numel(), dtype=torch.float32).pin_memory()
              for L_ in layers]
    dq = [torch.empty(t.shape, dtype=torch.int16, device=dev) for t in hq]
    dk = [torch.empty(t.shape, dtype=torch.int16, device=dev) for t in hk]
    dy = [torch.empty(t.shape, dtype=torch.int16, device=dev) for t in hy]
    dx = torch.empty(hx.shape, dtype=torch.int16, device=dev)
    stream = torch.cuda.current_stream(dev)
    h2d = sum(t.numel() * 2 for t in hq + hk + hy) + hx.numel() * 2
    d2h = hx_out.numel() * 2 + sum(t.numel() * 4 for t in hs_out)

    # Host -> device copies run on their own stream, ordered by events: layer
    # l + 1's inputs upload while layer l computes, and a layer's device
    # buffers are refilled only after the previous step's use of them.
    cs = torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    ready, used = [ev() for _ in range(nl)], [ev() for _ in range(nl)]
    x_ready, x_used = ev(), ev()
    for e in used + [x_used]:
        e.record(stream)

    def step():
        with torch.cuda.stream(cs):
            for l in range(nl):
                cs.wait_event(used[l])
                dq[l].copy_(hq[l], non_blocking=True)
                dk[l].copy_(hk[l], non_blocking=True)
                dy[l].copy_(hy[l], non_blocking=True)
                ready[l].record(cs)
                if l == 0:  # the residual stream right after the first layer's inputs
                    cs.wait_event(x_used)
                    dx.copy_(hx, non_blocking=True)
                    x_ready.record(cs)
        stream.wait_event(x_ready)
        for l in range(nl):
            stream.wait_event(ready[l])
            L_ = layers[l]
            L_.step(dq[l].view(torch.bfloat16), dk[l].view(torch.bfloat16), thetas[l],
                    dx.view(torch.bfloat16), dy[l].view(torch.bfloat16))
            used[l].record(stream)
            hs_out[l].copy_(L_.block_scores, non_blocking=True)
        hx_out.copy_(dx, non_blocking=True)
        x_used.record(stream)

    steps = max(3, min(args.steps, args.e2e_steps))
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier(world, local)
    torch.cuda.synchronize()
    a.record(stream)
    cs.wait_event(a)  # no copy of the timed steps starts before the clock
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world, local)
    s = max_over_ranks(a.elapsed_time(b) / 1e3, world, dev)
    return {"value": round(whole_job_rate(tokens_per_step, world, s / steps), 1), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "ms_per_step": round(1e3 * s / steps, 3),
            "path": "pinned host -> device copies (own stream, overlapping the previous layer), "
                    "lemo_* calls, device -> pinned host copies"}


# ----------------------------------------------------------------------------
# extension: segmented lm-head loss (segment-based peak cutting)
# ----------------------------------------------------------------------------

SEGLOSS_METRIC = "tokens/sec of the segmented lm-head loss (forward + backward)"


def run_segloss(args):
    import torch

    from contextual_token_sparsity_b200 import lemo, synth

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    lemo.load()
    cfg = synth.LM_HEAD_WORKLOADS[args.workload]
    T, d, V, S = cfg["T"], cfg["d"], cfg["V"], cfg["seg_rows"]
    h, w, y = synth.lm_head_inputs(T, d, V, cfg["seed"])
    hd = torch.from_numpy(h.view(np.int16)).to(dev)
    wd = torch.from_numpy(w.view(np.int16)).to(dev)
    yd = torch.from_numpy(y).to(dev)
    loss = torch.zeros(1, dtype=torch.float32, device=dev)
    dh = torch.empty((T, d), dtype=torch.int16, device=dev)
    dw = torch.zeros((V, d), dtype=torch.float32, device=dev)
    ws = torch.empty(lemo.lemo_segment_loss_workspace_size(T, V, S), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        lemo.lemo_segment_loss(hd, wd, yd, S, loss, ws, dh=dh, dw=dw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = lemo.lemo_get_error()
    if st != lemo.LEMO_OK:
        raise RuntimeError(f"device error during warm-up: {lemo.STATUS.get(st, st)}")
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(local)
    clocks = ClockSampler(gpu_id)
    clocks.start()
    time.sleep(0.3)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier(world, local)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world, local)
    elapsed = a.elapsed_time(b) / 1e3
    clk = clocks.stop()
    max_s = max_over_ranks(elapsed, world, dev)
    step_s = max_s / args.steps
    peaks = load_peaks()
    flops = 6.0 * T * V * d  # logits, dh and dW GEMMs
    peak_tf = peaks["bf16_tflops_sustained"] if elapsed > 2.0 else peaks["bf16_tflops"]
    ach = flops / step_s / 1e12
    full_ws = lemo.lemo_segment_loss_workspace_size(T, V, T)
    out = {
        "metric": SEGLOSS_METRIC, "value": round(whole_job_rate(T, world, step_s), 1),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_s * 1e3, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.workload}: Llama-2-7B lm head", "tokens": T, "d": d,
                   "vocab": V, "segment_rows": S, "segments": -(-T // S),
                   "l2": "not flushed; each step streams the 262 MB lm-head weight 48 times",
                   "parallelism": f"{world} independent replica(s), no collective"},
        "roofline": {"bound": "tensor", "kernel": "whole call (3 tcgen05 GEMMs + row kernel per "
                     "segment)", "achieved": round(ach, 1), "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": round(ach / peak_tf, 4), "traffic": None,
                     "algorithmic_flops_per_call": flops},
        "peak_memory": {"workspace_bytes": ws.numel(), "unsegmented_workspace_bytes": full_ws},
        "loss": float(loss.item()),
        # count + loss kernels; per segment the logits GEMM, the row kernel and
        # the dh GEMM; one dW GEMM per four segments
        "gpu_launches": (2 + 3 * -(-T // S) + -(-(-(-T // S)) // 4)) * args.steps,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = ext_cpu_baseline("lmhead-llama7b-16k", args.cpu_seconds)
    _finish(out, world, local, rank)


# ----------------------------------------------------------------------------
# extensions: attention over kept tokens, predicted path, MLP-block scores
# ----------------------------------------------------------------------------

ATTN_METRIC = "tokens/sec per layer of permutation-free attention over kept tokens"
PREDICT_METRIC = "tokens/sec per layer (predicted score+select+gather+scatter)"
MLP_METRIC = "tokens/sec per layer (MLP-block score+select+gather+scatter)"


def _setup_device(world, local):
    import torch
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(local)
    return dev, gpu_id


def _timed(step, steps, world, local, dev, gpu_id, n_marks=0):
    """Run `steps` calls of step(evs) between two events on the current
    stream (barrier + synchronize on both sides); step records its own
    per-part events into evs (a list of n_marks events per step).  Returns
    (elapsed seconds, clocks, per-step event lists)."""
    import torch
    stream = torch.cuda.current_stream(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_marks)] for _ in range(steps)]
    clocks = ClockSampler(gpu_id)
    clocks.start()
    time.sleep(0.3)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier(world, local)
    torch.cuda.synchronize()
    a.record(stream)
    for i in range(steps):
        step(ev[i])
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world, local)
    elapsed = a.elapsed_time(b) / 1e3
    return elapsed, clocks.stop(), ev


def _mean_us(ev, i0, i1):
    return 1e3 * statistics.fmean(e[i0].elapsed_time(e[i1]) for e in ev)


def _e2e(steps, world, local, dev, tokens, inputs, outputs, call):
    """The same work through the C ABI with host buffers: every step copies
    each (pinned host -> device) input pair in, runs call(), and copies each
    (device -> pinned host) output pair out."""
    import torch
    stream = torch.cuda.current_stream(dev)

    def step():
        for h, d in inputs:
            d.copy_(h, non_blocking=True)
        call()
        for d, h in outputs:
            h.copy_(d, non_blocking=True)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier(world, local)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world, local)
    s = max_over_ranks(a.elapsed_time(b) / 1e3, world, dev) / steps
    nb = lambda t: t.numel() * t.element_size()  # noqa: E731
    return {"value": round(whole_job_rate(tokens, world, s), 1), "unit": UNIT,
            "h2d_bytes_per_step": int(sum(nb(h) for h, _ in inputs)),
            "d2h_bytes_per_step": int(sum(nb(h) for _, h in outputs)), "steps": steps,
            "ms_per_step": round(1e3 * s, 3),
            "path": "pinned host -> device copies, lemo_* calls, device -> pinned host copies"}


def torch_empty_pinned(shape, dtype):
    import torch
    return torch.empty(shape, dtype=dtype).pin_memory()


_COLLECT = None  # a list while the headline run gathers the extension lines


def _finish(out, world, local, rank):
    if _COLLECT is not None:  # an extension run inside the headline run (one rank)
        _COLLECT.append(out)
        return
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def _header(metric, args, world, step_s, value):
    return {"metric": metric, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic"}


def attention_flops(kept_per_seq, H, dh) -> float:
    """Causal attention among K_s kept tokens: K_s (K_s + 1) / 2 query-key
    pairs per head, 2 dh flops for the score and 2 dh for P V."""
    return float(sum(2 * H * dh * K * (K + 1) for K in kept_per_seq))


def run_attention(args):
    """Attention over the kept tokens of the three llama7b-16k layers (keep 30/50/70 %),
    added in place into the residual stream.  The keep masks come from the
    path itself (score + select at set-up, with the stored thresholds)."""
    import torch

    from contextual_token_sparsity_b200 import lemo, synth
    from contextual_token_sparsity_b200.pipeline import Layer, to_device_bf16

    world, rank, local = dist_env()
    dev, gpu_id = _setup_device(world, local)
    lemo.load()
    key = "llama7b-16k"
    w = synth.WORKLOADS[key]
    nl = w.layers
    thetas = thresholds(key, nl)
    if thetas is None:
        raise RuntimeError("stored thresholds tests/golden/llama7b-16k.json are missing")
    hd = w.H * w.dh
    host = []
    for l in range(nl):
        inp = synth.make_workload(key, l, with_x=(l == 0))
        inp["v"] = synth.normal_bf16(w.total_L, hd, int(w.seeds[l]), 22)
        host.append(inp)
    hx = host[0]["x"][:, :hd]
    layers = [Layer(w.lengths, w.H, w.dh, w.block, hd, pad_to=PAD_TO, device=dev)
              for _ in range(nl)]
    q = [to_device_bf16(h["q"], dev) for h in host]
    k = [to_device_bf16(h["k"], dev) for h in host]
    v = [to_device_bf16(h["v"], dev) for h in host]
    x = to_device_bf16(np.ascontiguousarray(hx), dev)
    for l in range(nl):
        layers[l].score(q[l], k[l])
        layers[l].select(thetas[l])
    ws = [torch.empty(lemo.lemo_attention_workspace_size(len(w.lengths)), dtype=torch.uint8,
                      device=dev) for _ in range(nl)]
    torch.cuda.synchronize()
    cu_k = [L_.cu_kept.cpu().numpy() for L_ in layers]
    kept_seq = [np.diff(c).tolist() for c in cu_k]
    kept = [int(c[-1]) for c in cu_k]

    def call(xx, qq=q, kk=k, vv=v, evs=None):
        for l in range(nl):
            if evs is not None:
                evs[l].record()
            L_ = layers[l]
            lemo.lemo_attention_kept(L_.shape, qq[l], kk[l], vv[l], L_.kept_idx, L_.cu_kept,
                                     L_.kept_total, ws[l], x=xx)
        if evs is not None:
            evs[nl].record()

    for _ in range(args.warmup):
        call(x)
    torch.cuda.synchronize()
    st = lemo.lemo_get_error()
    if st != lemo.LEMO_OK:
        raise RuntimeError(f"device error during warm-up: {lemo.STATUS.get(st, st)}")
    elapsed, clk, ev = _timed(lambda e: call(x, evs=e), args.steps, world, local, dev, gpu_id,
                              nl + 1)
    st = lemo.lemo_get_error()
    if st != lemo.LEMO_OK:
        raise RuntimeError(f"device error in timed region: {lemo.STATUS.get(st, st)}")
    step_s = max_over_ranks(elapsed, world, dev) / args.steps
    per_layer_us = [_mean_us(ev, l, l + 1) for l in range(nl)]
    peaks = load_peaks()
    peak_tf = peaks["bf16_tflops_sustained"] if elapsed > 2.0 else peaks["bf16_tflops"]
    flops = [attention_flops(kept_seq[l], w.H, w.dh) for l in range(nl)]
    ach = [flops[l] / (per_layer_us[l] * 1e-6) / 1e12 for l in range(nl)]
    tot_f = sum(flops)
    tot_ach = tot_f / (sum(per_layer_us) * 1e-6) / 1e12
    out = _header(ATTN_METRIC, args, world, step_s, whole_job_rate(nl * w.total_L, world, step_s))
    out["config"] = {"workload": f"attn-llama7b-16k: attention over the kept tokens of the {key} "
                                 f"layers (L={w.total_L}, H={w.H}, dh={w.dh}, b={w.block}, keep "
                                 f"30/50/70%), output added into the residual in place",
                     "layers": nl, "kept_tokens": kept, "softmax_scale": "1/sqrt(dh)",
                     "l2": "not flushed; each step reads 3 x 3 x 134 MB of Q/K/V rows "
                           "(> 126 MB L2)",
                     "parallelism": f"{world} independent replica(s), no collective"}
    out["roofline"] = {"bound": "tensor", "kernel": "attn_kernel (+plan)",
                       "achieved": round(tot_ach, 1), "peak": peak_tf, "unit": "TFLOP/s",
                       "frac": round(tot_ach / peak_tf, 4), "traffic": None,
                       "peak_source": f"{peaks['source']} bf16 "
                                      f"{'sustained' if elapsed > 2.0 else 'burst'} cuBLAS GEMM",
                       "algorithmic_flops_per_step": tot_f,
                       "per_layer": [{"K": kept[l], "us": round(per_layer_us[l], 2),
                                      "tflops": round(ach[l], 1)} for l in range(nl)]}
    out["gpu_launches"] = 2 * nl * args.steps
    out["clocks"] = clk
    if not args.no_e2e:
        pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()  # noqa
        hq, hk, hv = ([pin(h[n]) for h in host] for n in ("q", "k", "v"))
        hxp = pin(hx)
        hx_out = torch_empty_pinned(hxp.shape, hxp.dtype)
        dq = [torch.empty(t.shape, dtype=torch.int16, device=dev) for t in hq]
        dk = [torch.empty(t.shape, dtype=torch.int16, device=dev) for t in hk]
        dv = [torch.empty(t.shape, dtype=torch.int16, device=dev) for t in hv]
        dx = torch.empty(hxp.shape, dtype=torch.int16, device=dev)
        bf = lambda ts: [t.view(torch.bfloat16) for t in ts]  # noqa: E731
        out["e2e"] = _e2e(max(3, min(args.steps, args.e2e_steps)), world, local, dev,
                          nl * w.total_L,
                          list(zip(hq, dq)) + list(zip(hk, dk)) + list(zip(hv, dv)) + [(hxp, dx)],
                          [(dx, hx_out)],
                          lambda: call(dx.view(torch.bfloat16), bf(dq), bf(dk), bf(dv)))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = ext_cpu_baseline("attn-llama7b-16k", args.cpu_seconds)
    _finish(out, world, local, rank)


SPLIT_METRIC = "tokens/sec per layer (score+select+gather+scatter), one sequence split over the GPUs"


def run_split(args):
    """One long sequence split over the ranks (strong scaling): each rank
    scores the key blocks of its key tiles (lemo_score_blocks_shard), one
    all-reduce of the block scores gives every rank the full scores, and each
    rank selects, gathers and scatters the kept rows of its own token shard.
    Q and K are replicated on every rank; the residual and the sublayer output
    are sharded by tokens."""
    import torch

    from contextual_token_sparsity_b200 import lemo, split, synth
    from contextual_token_sparsity_b200.pipeline import to_device_bf16

    world, rank, local = dist_env()
    dev, gpu_id = _setup_device(world, local)
    lemo.load()
    w = synth.WORKLOADS[args.workload]
    if len(w.lengths) != 1:
        raise ValueError("--split-sequence takes a workload of one sequence")
    nl, L = w.layers, w.total_L
    thetas = thresholds(args.workload, nl)
    if thetas is None:
        raise RuntimeError(f"stored thresholds tests/golden/{args.workload}.json are missing")
    host = [synth.make_workload(args.workload, l, with_x=True) for l in range(nl)]
    layers = [split.SplitLayer(L, w.H, w.dh, w.block, w.d, rank, world, pad_to=PAD_TO, device=dev)
              for _ in range(nl)]
    lo, hi = layers[0].lo, layers[0].hi
    q = [to_device_bf16(h["q"], dev) for h in host]
    k = [to_device_bf16(h["k"], dev) for h in host]
    y = [to_device_bf16(np.ascontiguousarray(h["y_out"][lo:hi]), dev) for h in host]
    x = to_device_bf16(np.ascontiguousarray(host[0]["x"][lo:hi]), dev)

    def step(evs=None, qq=q, kk=k, xx=x, yy=y):
        for l in range(nl):
            sl = layers[l]
            if evs is not None:
                evs[4 * l].record()
            sl.score(qq[l], kk[l])
            if evs is not None:
                evs[4 * l + 1].record()
            sl.select(thetas[l])
            if evs is not None:
                evs[4 * l + 2].record()
            sl.gather(xx)
            sl.scatter(xx, yy[l])
            if evs is not None:
                evs[4 * l + 3].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = lemo.lemo_get_error()
    if st != lemo.LEMO_OK:
        raise RuntimeError(f"device error during warm-up: {lemo.STATUS.get(st, st)}")
    kept_local = [int(sl.kept_total.item()) for sl in layers]
    elapsed, clk, ev = _timed(step, args.steps, world, local, dev, gpu_id, 4 * nl)
    st = lemo.lemo_get_error()
    if st != lemo.LEMO_OK:
        raise RuntimeError(f"device error in timed region: {lemo.STATUS.get(st, st)}")
    step_s = max_over_ranks(elapsed, world, dev) / args.steps
    us = {"score+allreduce": statistics.fmean(_mean_us(ev, 4 * l, 4 * l + 1) for l in range(nl)),
          "select": statistics.fmean(_mean_us(ev, 4 * l + 1, 4 * l + 2) for l in range(nl)),
          "gather+scatter": statistics.fmean(_mean_us(ev, 4 * l + 2, 4 * l + 3)
                                             for l in range(nl))}
    kept_all = [int(sl.offsets()[-1].item()) for sl in layers]
    out = _header(SPLIT_METRIC, args, world, step_s, nl * L / step_s)
    out["scaling"] = "strong"
    out["config"] = {"workload": f"{args.workload}: {w.name}", "layers": nl, "seq_lens": [L],
                     "heads": w.H, "head_dim": w.dh, "block": w.block, "d": w.d,
                     "keep": list(w.keep), "kept_tokens": kept_all,
                     "kept_tokens_this_rank": kept_local, "token_shard": [lo, hi],
                     "parallelism": f"one sequence over {world} rank(s): key-tile shards of the "
                                    "scoring (snake order), one all-reduce of the block scores "
                                    "per layer, token shards of the movement; Q and K replicated",
                     "l2": "not flushed; each step streams "
                           f"{nl * 2 * L * w.H * w.dh * 2 / 1e9:.2f} GB of Q/K (> 126 MB L2)"}
    out["kernels_us"] = {k_: round(v, 2) for k_, v in us.items()}
    out["gpu_launches"] = 7 * nl * args.steps
    out["clocks"] = clk
    if not args.no_e2e:
        pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()  # noqa
        hq = [pin(h["q"]) for h in host]
        hk = [pin(h["k"]) for h in host]
        hy = [pin(h["y_out"][lo:hi]) for h in host]
        hx = pin(host[0]["x"][lo:hi])
        hx_out = torch_empty_pinned(hx.shape, hx.dtype)
        dq = [torch.empty(t.shape, dtype=torch.int16, device=dev) for t in hq]
        dk = [torch.empty(t.shape, dtype=torch.int16, device=dev) for t in hk]
        dy = [torch.empty(t.shape, dtype=torch.int16, device=dev) for t in hy]
        dx = torch.empty(hx.shape, dtype=torch.int16, device=dev)
        bf = lambda ts: [t.view(torch.bfloat16) for t in ts]  # noqa: E731
        out["e2e"] = _e2e(max(3, min(args.steps, args.e2e_steps)), world, local, dev, nl * L / world,
                          list(zip(hq, dq)) + list(zip(hk, dk)) + list(zip(hy, dy)) + [(hx, dx)],
                          [(dx, hx_out)],
                          lambda: step(None, bf(dq), bf(dk), dx.view(torch.bfloat16), bf(dy)))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.workload, budget_s=args.cpu_seconds)
    _finish(out, world, local, rank)


def run_predict(args):
    """The predicted path at the Llama-2-13B layer (llama13b-32k): block means of X,
    the two rank-256 ReLU predictors (pruned neurons left out: rank 154),
    block products and column sums, then select / gather / scatter with the
    stored predicted-score threshold."""
    import torch

    from contextual_token_sparsity_b200 import lemo, synth
    from contextual_token_sparsity_b200.pipeline import Layer, to_device_bf16

    world, rank, local = dist_env()
    dev, gpu_id = _setup_device(world, local)
    lemo.load()
    key = "llama13b-32k"
    w = synth.WORKLOADS[key]
    seed = int(w.seeds[0])
    path = os.path.join(ROOT, "tests", "golden", f"{key}.json")
    if not os.path.exists(path):
        raise RuntimeError("stored thresholds tests/golden/llama13b-32k.json are missing")
    with open(path) as f:
        theta = float(json.load(f)["layers"][0]["pred_theta"])
    L, d, hd = w.total_L, w.d, w.H * w.dh
    xb, _ = synth.projected_x(L, d, float(w.salient), seed)
    w1q, w2q, liveq = synth.predictor_weights(d, w.predictor_rank, hd, 0.4, seed, 10)
    w1k, w2k, livek = synth.predictor_weights(d, w.predictor_rank, hd, 0.4, seed, 11)
    w1q, w2q = np.ascontiguousarray(w1q[:, liveq]), np.ascontiguousarray(w2q[liveq])
    w1k, w2k = np.ascontiguousarray(w1k[:, livek]), np.ascontiguousarray(w2k[livek])
    y_out = synth.normal_bf16(L, d, seed, 8)
    layer = Layer(w.lengths, w.H, w.dh, w.block, d, pad_to=PAD_TO, device=dev)
    x = to_device_bf16(xb, dev)
    dw = [to_device_bf16(a, dev) for a in (w1q, w2q, w1k, w2k)]
    yd = to_device_bf16(y_out, dev)
    rank_eff = int(w1q.shape[1])
    pws = torch.empty(lemo.lemo_predict_workspace_size(layer.shape, d, rank_eff),
                      dtype=torch.uint8, device=dev)

    def call(xx, yy, evs=None):
        if evs is not None:
            evs[0].record()
        lemo.lemo_predict_scores(layer.shape, xx, *dw, layer.block_scores, pws)
        if evs is not None:
            evs[1].record()
        layer.select(theta)
        if evs is not None:
            evs[2].record()
        layer.gather(xx)
        if evs is not None:
            evs[3].record()
        layer.scatter(xx, yy)
        if evs is not None:
            evs[4].record()

    for _ in range(args.warmup):
        call(x, yd)
    torch.cuda.synchronize()
    st = lemo.lemo_get_error()
    if st != lemo.LEMO_OK:
        raise RuntimeError(f"device error during warm-up: {lemo.STATUS.get(st, st)}")
    K = int(layer.kept_total.item())
    elapsed, clk, ev = _timed(lambda e: call(x, yd, e), args.steps, world, local, dev, gpu_id, 5)
    st = lemo.lemo_get_error()
    if st != lemo.LEMO_OK:
        raise RuntimeError(f"device error in timed region: {lemo.STATUS.get(st, st)}")
    step_s = max_over_ranks(elapsed, world, dev) / args.steps
    us = {n: _mean_us(ev, i, i + 1) for i, n in enumerate(("predict", "select", "gather",
                                                              "scatter"))}
    peaks = load_peaks()
    pool_bytes = 2 * L * d  # X read once for the block means
    g_b, s_b = move_bytes(K, d)
    tb = -(-L // w.block)
    pred_flops = 2 * 2 * tb * (d * rank_eff + rank_eff * hd) + tb * (tb + 1) * hd
    bw = peaks["hbm_gbs"]
    out = _header(PREDICT_METRIC, args, world, step_s, whole_job_rate(L, world, step_s))
    out["config"] = {"workload": f"predict-llama13b-32k: {w.name}", "seq_lens": list(w.lengths),
                     "heads": w.H, "head_dim": w.dh, "block": w.block, "d": d,
                     "predictor_rank": w.predictor_rank, "live_neurons": [len(liveq), len(livek)],
                     "keep": 0.5, "kept_tokens": K, "threshold_source":
                     "oracle predicted scores (tests/golden)",
                     "l2": "not flushed; each step reads the 335 MB X twice (> 126 MB L2)",
                     "parallelism": f"{world} independent replica(s), no collective"}
    pred_gbs = pool_bytes / (us["predict"] * 1e-6) / 1e9
    out["roofline"] = {"bound": "hbm", "kernel": "lemo_predict_scores (pool + predictor GEMMs "
                       "+ block products + column sum)", "achieved": round(pred_gbs, 1),
                       "peak": bw, "unit": "GB/s", "frac": round(pred_gbs / bw, 4),
                       "traffic": None, "algorithmic_bytes_per_call": pool_bytes,
                       "predictor_flops_per_call": pred_flops}
    out["kernels_us"] = {n: round(v, 2) for n, v in us.items()}
    out["movement"] = {"gather_gbs": round(g_b / (us["gather"] * 1e-6) / 1e9, 1),
                       "scatter_gbs": round(s_b / (us["scatter"] * 1e-6) / 1e9, 1),
                       "hbm_peak_gbs": bw}
    # predict: (plan,) pooling pass, persistent predictor kernel - a batch of
    # one sequence has its plan written by the pooling pass; select: plan,
    # select; gather; scatter
    out["gpu_launches"] = ((2 if len(w.lengths) == 1 else 3) + 4) * args.steps
    out["clocks"] = clk
    if not args.no_e2e:
        pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()  # noqa
        hxp, hyp = pin(xb), pin(y_out)
        hx_out = torch_empty_pinned(hxp.shape, hxp.dtype)
        hs = torch_empty_pinned(layer.block_scores.shape, torch.float32)
        dx = torch.empty(hxp.shape, dtype=torch.int16, device=dev)
        dy = torch.empty(hyp.shape, dtype=torch.int16, device=dev)
        out["e2e"] = _e2e(max(3, min(args.steps, args.e2e_steps)), world, local, dev, L,
                          [(hxp, dx), (hyp, dy)], [(dx, hx_out), (layer.block_scores, hs)],
                          lambda: call(dx.view(torch.bfloat16), dy.view(torch.bfloat16)))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = ext_cpu_baseline("predict-llama13b-32k", args.cpu_seconds)
    _finish(out, world, local, rank)


def run_mlp(args):
    """MLP-block elimination at the Llama-2-7B layer (L = 16384, SiLU-gated
    d_ff = 11008, b = 64): token scores from SiLU(gate) * up, block maxima,
    keep mask at 50 %, gather / scatter of d = 4096 rows."""
    import torch

    from contextual_token_sparsity_b200 import lemo, synth
    from contextual_token_sparsity_b200.pipeline import Layer, to_device_bf16

    world, rank, local = dist_env()
    dev, gpu_id = _setup_device(world, local)
    lemo.load()
    L, d_ff, d, b, seed = 16384, 11008, 4096, 64, 0
    gate, up = synth.mlp_activations(L, d_ff, 0.1, seed=seed, gated=True)
    xb = synth.normal_bf16(L, d, seed, 7)
    y_out = synth.normal_bf16(L, d, seed, 8)
    layer = Layer([L], 1, 64, b, d, pad_to=PAD_TO, device=dev)
    g_d, u_d = to_device_bf16(gate, dev), to_device_bf16(up, dev)
    x, yd = to_device_bf16(xb, dev), to_device_bf16(y_out, dev)
    lemo.lemo_mlp_block_scores(layer.shape, layer.block_scores, layer.ws, gate=g_d, up=u_d)
    s = np.sort(layer.block_scores[: layer.total_blocks].cpu().numpy().astype(np.float64))[::-1]
    kk = int(math.floor(0.5 * s.size + 0.5))
    theta = float(0.5 * (s[kk - 1] + s[kk]))

    def call(gg, uu, xx, yy, evs=None):
        if evs is not None:
            evs[0].record()
        lemo.lemo_mlp_block_scores(layer.shape, layer.block_scores, layer.ws, gate=gg, up=uu)
        if evs is not None:
            evs[1].record()
        layer.select(theta)
        if evs is not None:
            evs[2].record()
        layer.gather(xx)
        if evs is not None:
            evs[3].record()
        layer.scatter(xx, yy)
        if evs is not None:
            evs[4].record()

    for _ in range(args.warmup):
        call(g_d, u_d, x, yd)
    torch.cuda.synchronize()
    st = lemo.lemo_get_error()
    if st != lemo.LEMO_OK:
        raise RuntimeError(f"device error during warm-up: {lemo.STATUS.get(st, st)}")
    K = int(layer.kept_total.item())
    elapsed, clk, ev = _timed(lambda e: call(g_d, u_d, x, yd, e), args.steps, world, local, dev,
                              gpu_id, 5)
    st = lemo.lemo_get_error()
    if st != lemo.LEMO_OK:
        raise RuntimeError(f"device error in timed region: {lemo.STATUS.get(st, st)}")
    step_s = max_over_ranks(elapsed, world, dev) / args.steps
    us = {n: _mean_us(ev, i, i + 1) for i, n in enumerate(("mlp_score", "select", "gather",
                                                              "scatter"))}
    peaks = load_peaks()
    bw = peaks["hbm_gbs"]
    score_bytes = 4 * L * d_ff  # gate and up read once
    gbs = score_bytes / (us["mlp_score"] * 1e-6) / 1e9
    g_b, s_b = move_bytes(K, d)
    out = _header(MLP_METRIC, args, world, step_s, whole_job_rate(L, world, step_s))
    out["config"] = {"workload": f"mlp-llama7b-16k: L={L}, SiLU-gated d_ff={d_ff}, b={b}, d={d}, "
                                 "keep 50%", "kept_tokens": K,
                     "threshold_source": "keep ratio on the kernel's own block scores",
                     "l2": "not flushed; each step reads 721 MB of activations (> 126 MB L2)",
                     "parallelism": f"{world} independent replica(s), no collective"}
    out["roofline"] = {"bound": "hbm", "kernel": "mlp::block_scores_kernel (+plan, column "
                       "max)", "achieved": round(gbs, 1), "peak": bw, "unit": "GB/s",
                       "frac": round(gbs / bw, 4), "traffic": None,
                       "algorithmic_bytes_per_call": score_bytes}
    out["kernels_us"] = {n: round(v, 2) for n, v in us.items()}
    out["movement"] = {"gather_gbs": round(g_b / (us["gather"] * 1e-6) / 1e9, 1),
                       "scatter_gbs": round(s_b / (us["scatter"] * 1e-6) / 1e9, 1),
                       "hbm_peak_gbs": bw}
    out["gpu_launches"] = 6 * args.steps  # plan + scores, plan + select, gather, scatter
    out["clocks"] = clk
    if not args.no_e2e:
        pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()  # noqa
        hg, hu, hxp, hyp = pin(gate), pin(up), pin(xb), pin(y_out)
        hx_out = torch_empty_pinned(hxp.shape, hxp.dtype)
        dd = [torch.empty(t.shape, dtype=torch.int16, device=dev) for t in (hg, hu, hxp, hyp)]
        out["e2e"] = _e2e(max(3, min(args.steps, args.e2e_steps)), world, local, dev, L,
                          list(zip((hg, hu, hxp, hyp), dd)), [(dd[2], hx_out)],
                          lambda: call(*[t.view(torch.bfloat16) for t in dd]))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = ext_cpu_baseline("mlp-llama7b-16k", args.cpu_seconds)
    _finish(out, world, local, rank)


# ----------------------------------------------------------------------------
# the CPU oracle (cpu_baseline leg and reference arm)
# ----------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


class OracleSample:
    """The CPU oracle on a bounded sample of one layer, scaled to tokens/s.

    The oracle scores one query-block row at a time; a sample is a set of
    query-block rows drawn at random until a time budget is spent.  A row's
    cost is proportional to its number of key blocks (n + 1), so the full
    layer's scoring time is the sample time times (all block pairs / sampled
    block pairs).  Selection, compaction, gather and scatter run in full.
    """

    def __init__(self, key: str, layer: int = 0):
        import oracle
        from contextual_token_sparsity_b200 import synth
        self.oracle = oracle
        self.key, self.layer = key, layer
        self.w = w = synth.WORKLOADS[key]
        self.inp = inp = synth.make_workload(key, layer, with_x=True)
        cu = inp["cu_seqlens"]
        s = int(np.argmax(w.lengths))  # sample rows from the longest sequence
        L = w.lengths[s]
        self.q = oracle.bf16_bits_to_f64(inp["q"][cu[s]:cu[s + 1]]).reshape(L, w.H, w.dh)
        self.k = oracle.bf16_bits_to_f64(inp["k"][cu[s]:cu[s + 1]]).reshape(L, w.H, w.dh)
        self.nb = -(-L // w.block)
        self.all_pairs = sum((-(-Ls // w.block)) * ((-(-Ls // w.block)) + 1) // 2
                             for Ls in w.lengths)
        self.t_rest = None

    def time_rows(self, budget_s: float, seed: int):
        order = np.random.default_rng(seed).permutation(self.nb)
        t0 = time.perf_counter()
        pairs = rows = 0
        for n in order:
            self.oracle.block_max_row(self.q, self.k, int(n), self.w.block)
            pairs += int(n) + 1
            rows += 1
            if time.perf_counter() - t0 > budget_s:
                break
        t = time.perf_counter() - t0
        return t * self.all_pairs / pairs, rows, pairs, t

    def run_rest(self):
        """select + compact + gather + scatter of the layer, in full; returns
        its time."""
        o, w, inp = self.oracle, self.w, self.inp
        gpath = os.path.join(ROOT, "tests", "golden", f"{self.key}.json")
        if os.path.exists(gpath):
            with open(gpath) as f:
                g = json.load(f)["layers"][self.layer]
            sc = np.array([float(v) for v in g["scores"]])
            theta = float(g["theta"])
        else:
            sc = np.linspace(1.0, 0.0, sum(-(-Ls // w.block) for Ls in w.lengths))
            theta = 0.5
        t1 = time.perf_counter()
        mask = o.keep_mask(sc, theta)
        idx, _, _ = o.compact(mask, inp["cu_seqlens"], w.block)
        o.gather_pad(inp["x"], idx, PAD_TO)
        o.scatter_residual(inp["x"], inp["y_out"], idx)
        self.t_rest = time.perf_counter() - t1
        return self.t_rest

    def time_rest(self):
        """select + compact + gather + scatter of the layer, in full (timed once)."""
        return self.t_rest if self.t_rest is not None else self.run_rest()

    def describe(self, rows, pairs, t_rows):
        return (f"layer {self.layer} of {self.key}: {rows} of {self.nb} query-block rows "
                f"({pairs} of {self.all_pairs} block pairs, {t_rows:.1f} s) scored by the "
                f"oracle and scaled by block pairs; select/compact/gather/scatter timed in "
                f"full ({self.t_rest:.1f} s); float64 numpy, BLAS on all cores, elementwise "
                f"work single-threaded")


def cpu_baseline(key: str, budget_s: float = 20.0, layer: int = 0):
    smp = OracleSample(key, layer)
    t_rest = smp.time_rest()
    t_score, rows, pairs, t_rows = smp.time_rows(budget_s, seed=0)
    t_layer = t_score + t_rest
    return {"value": round(smp.w.total_L / t_layer, 3), "unit": UNIT, "cores": blas_threads(),
            "kind": "oracle", "sample": smp.describe(rows, pairs, t_rows),
            "seconds_per_layer_estimate": round(t_layer, 2)}


def oracle_sample(workload: str, budget_s: float = 20.0, seed: int = 0):
    """The CPU oracle, as it stands, on a bounded sample of an extension
    workload.  Returns (estimated seconds per layer / call, tokens it covers,
    description of the sample)."""
    import oracle
    from contextual_token_sparsity_b200 import synth
    rng = np.random.default_rng(seed)
    if workload == "predict-llama13b-32k":
        w = synth.WORKLOADS["llama13b-32k"]
        sd, L, d, hd = int(w.seeds[0]), w.total_L, w.d, w.H * w.dh
        with open(os.path.join(ROOT, "tests", "golden", "llama13b-32k.json")) as f:
            theta = float(json.load(f)["layers"][0]["pred_theta"])
        xb, _ = synth.projected_x(L, d, float(w.salient), sd)
        w1q, w2q, lq = synth.predictor_weights(d, w.predictor_rank, hd, 0.4, sd, 10)
        w1k, w2k, lk = synth.predictor_weights(d, w.predictor_rank, hd, 0.4, sd, 11)
        y = synth.normal_bf16(L, d, sd, 8)
        cu = np.array([0, L], dtype=np.int32)
        t0 = time.perf_counter()
        reps = oracle.block_representatives(xb, cu, w.block)
        qh = oracle.predictor_embeddings(reps, w1q[:, lq], w2q[lq])
        kh = oracle.predictor_embeddings(reps, w1k[:, lk], w2k[lk])
        _, ps = oracle.predict_scores(qh, kh, cu, w.block, w.H, w.dh)
        idx, _, _ = oracle.compact(oracle.keep_mask(ps, theta), cu, w.block)
        oracle.gather_pad(xb, idx, PAD_TO)
        oracle.scatter_residual(xb, y, idx)
        t = time.perf_counter() - t0
        return t, L, (f"predict-llama13b-32k in full ({t:.1f} s): block means, both predictors, "
                      "Eq. 3 block products, threshold, compaction, gather and scatter; float64 numpy")
    if workload == "attn-llama7b-16k":
        w = synth.WORKLOADS["llama7b-16k"]
        with open(os.path.join(ROOT, "tests", "golden", "llama7b-16k.json")) as f:
            g = json.load(f)["layers"][1]
        inp = synth.make_workload("llama7b-16k", 1, with_x=False)
        hd = w.H * w.dh
        v = synth.normal_bf16(w.total_L, hd, int(w.seeds[1]), 22)
        mask = oracle.keep_mask(np.array([float(x) for x in g["scores"]]), float(g["theta"]))
        idx, cu_k, K = oracle.compact(mask, inp["cu_seqlens"], w.block)
        order = rng.permutation(K)
        t0 = time.perf_counter()
        pairs = rows = 0
        for r in order:
            oracle.attention_kept_rows(inp["q"], inp["k"], v, idx[:K], cu_k, w.H, w.dh, [int(r)])
            pairs += int(r) + 1
            rows += 1
            if time.perf_counter() - t0 > budget_s:
                break
        t = time.perf_counter() - t0
        all_pairs = K * (K + 1) // 2
        return t * all_pairs / pairs, w.total_L, (
            f"layer 1 of attn-llama7b-16k (K = {K}): {rows} of {K} query rows "
            f"({pairs} of {all_pairs} query-key pairs, {t:.1f} s) by the oracle, scaled by pairs; float64 numpy")
    if workload == "mlp-llama7b-16k":
        L, d_ff, d, b = 16384, 11008, 4096, 64
        gate, up = synth.mlp_activations(L, d_ff, 0.1, seed=0, gated=True)
        chunk, t_sc, done = 512, 0.0, 0
        while done < L and t_sc < budget_s:
            t0 = time.perf_counter()
            oracle.mlp_token_scores(gate_bits=gate[done:done + chunk], up_bits=up[done:done + chunk])
            t_sc += time.perf_counter() - t0
            done += chunk
        cu = np.array([0, L], dtype=np.int32)
        x, y = synth.normal_bf16(L, d, 0, 7), synth.normal_bf16(L, d, 0, 8)
        t0 = time.perf_counter()
        bs = oracle.mlp_block_scores(np.linspace(1.0, 0.0, L), cu, b)  # costs do not depend on values
        idx, _, _ = oracle.compact(oracle.keep_mask(bs, float(np.median(bs))), cu, b)
        oracle.gather_pad(x, idx, PAD_TO)
        oracle.scatter_residual(x, y, idx)
        t_rest = time.perf_counter() - t0
        return t_sc * L / done + t_rest, L, (
            f"mlp-llama7b-16k: token scores of {done} of {L} tokens ({t_sc:.1f} s) scaled by "
            f"tokens; block scores, threshold, compaction, gather and scatter in full ({t_rest:.1f} s); float64 numpy")
    if workload == "lmhead-llama7b-16k":
        cfg = synth.LM_HEAD_WORKLOADS["lmhead-llama7b-16k"]
        T, d, V = cfg["T"], cfg["d"], cfg["V"]
        h, wt, y = synth.lm_head_inputs(T, d, V, cfg["seed"])
        R = 64
        t0 = time.perf_counter()
        oracle.lm_head_loss(h[:R], wt, y[:R])
        t = time.perf_counter() - t0
        return t * T / R, T, (f"lmhead-llama7b-16k: the oracle's full definition (logits, loss, "
                              f"dh and dW) on the first {R} of {T} tokens ({t:.1f} s), scaled by tokens; float64 numpy")
    raise ValueError(workload)


def ext_cpu_baseline(workload: str, budget_s: float):
    t, tokens, desc = oracle_sample(workload, budget_s)
    return {"value": round(tokens / t, 3), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": desc, "seconds_per_layer_estimate": round(t, 2)}


def run_reference_ext(args):
    world, rank, local = dist_env()
    if rank != 0:
        return  # the reference arm runs on rank 0 only
    per_step = max(0.3, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    vals, desc, tokens = [], "", 0
    for i in range(args.warmup + args.steps):
        t, tokens, d = oracle_sample(args.workload, per_step, seed=i)
        if i >= args.warmup:
            vals.append(t)
            desc = d
    t = statistics.fmean(vals)
    value = tokens / t
    metric = {"attn-llama7b-16k": ATTN_METRIC, "predict-llama13b-32k": PREDICT_METRIC,
              "mlp-llama7b-16k": MLP_METRIC, "lmhead-llama7b-16k": SEGLOSS_METRIC}[args.workload]
    out = {
        "metric": metric, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": args.workload, "parallelism": "CPU oracle, rank 0 only"},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": blas_threads(),
                         "kind": "oracle", "sample": f"per step: {desc}"},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def golden_kept(key: str, w, thetas):
    """Kept tokens per layer from the stored oracle scores and thresholds."""
    import oracle
    with open(os.path.join(ROOT, "tests", "golden", f"{key}.json")) as f:
        g = json.load(f)
    cu = np.zeros(len(w.lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(w.lengths)
    kept = []
    for l in range(w.layers):
        sc = np.array([float(v) for v in g["layers"][l]["scores"]])
        _, _, K = oracle.compact(oracle.keep_mask(sc, thetas[l]), cu, w.block)
        kept.append(int(K))
    return kept


def run_reference(args):
    """The reference arm: the CPU oracle, as it stands, on a bounded sample of
    the workload per step.  A step scores a random set of query-block rows of
    layer 0 for a fixed time budget and runs threshold, compaction, gather and
    scatter of that layer in full; ms_per_step is the measured time of that
    sampled work.  `value` scales the sample to a whole layer by block pairs
    (a row's cost is proportional to its key blocks) and is reported in the
    headline's unit, with the scale factor beside it."""
    world, rank, local = dist_env()
    if rank != 0:
        return  # the reference arm runs on rank 0 only
    from contextual_token_sparsity_b200 import synth
    w = synth.WORKLOADS[args.workload]
    thetas = thresholds(args.workload, w.layers)
    smp = OracleSample(args.workload, 0)
    per_step = max(0.3, min(20.0, 90.0 / max(1, args.steps + args.warmup)))
    measured, layer_est, fracs, desc = [], [], [], ""
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        t_score, rows, pairs, t_rows = smp.time_rows(per_step, seed=i)
        t_rest = smp.run_rest()
        t_step = time.perf_counter() - t0
        if i >= args.warmup:
            measured.append(t_step)
            layer_est.append(t_score + t_rest)
            fracs.append(pairs / smp.all_pairs)
            desc = smp.describe(rows, pairs, t_rows)
    t_layer = statistics.fmean(layer_est)
    value = w.total_L / t_layer
    if thetas is not None:
        kept, theta_src = golden_kept(args.workload, w, thetas), "oracle scores (tests/golden)"
    else:
        kept, theta_src = [], "none stored"
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * statistics.fmean(measured), 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": headline_config(args.workload, w, kept, thetas, theta_src, world),
        "reference_arm": "CPU oracle on rank 0 only (the other ranks exit without work); "
                         "each step is a bounded sample of layer 0",
        "sample": {"block_pair_fraction_per_step": round(statistics.fmean(fracs), 4),
                   "measured_s_per_step": round(statistics.fmean(measured), 2),
                   "extrapolated_s_per_layer": round(t_layer, 2),
                   "extrapolated_ms_per_full_step": round(1e3 * t_layer * w.layers, 1)},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": blas_threads(),
                         "kind": "oracle", "sample": f"per step: {desc}"},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description="contextual token sparsity hot-path benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["lemo", "reference"], default="lemo")
    ap.add_argument("--workload", default="llama7b-16k",
                    choices=["small-1k", "llama7b-8k", "llama7b-16k", "varlen-10k", "llama13b-32k",
                             "lmhead-llama7b-16k", "attn-llama7b-16k", "predict-llama13b-32k",
                             "mlp-llama7b-16k"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-extensions", action="store_true",
                    help="skip the short runs of the extension workloads in the headline line")
    ap.add_argument("--split-sequence", action="store_true",
                    help="split each sequence over the ranks (strong scaling) instead of one "
                         "replica per rank")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = dist_env()[0]
    if args.gpus != world and world > 1:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    extensions = {"lmhead-llama7b-16k": run_segloss, "attn-llama7b-16k": run_attention,
                  "predict-llama13b-32k": run_predict, "mlp-llama7b-16k": run_mlp}
    if args.workload in extensions:
        if args.impl == "reference":
            run_reference_ext(args)
        else:
            extensions[args.workload](args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.split_sequence:
        run_split(args)
    else:
        run_lemo(args)


if __name__ == "__main__":
    main()

"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

With N ranks every rank runs its own copy of the workload (independent layers,
no data-path collective).  The only cross-rank step is the timing reduction:
the step time is the maximum over ranks and the throughput counts every
rank's tokens.  These tests run that logic in two gloo processes.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, l = bench.dist_env()
        assert (w, r, l) == (world, rank, rank)
        elapsed = 1.0 + rank  # rank 1 is the slow one
        bench.barrier(world, l, cuda=False)
        m = bench.max_over_ranks(elapsed, world, None)
        rate = bench.whole_job_rate(3 * 16384, world, m)
        out.put((rank, m, rate))
        bench.barrier(world, l, cuda=False)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_max_time_and_count_all_tokens():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=10) for _ in range(world))
    for rank, m, rate in res:
        assert m == pytest.approx(2.0)
        assert rate == pytest.approx(2 * 3 * 16384 / 2.0)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(100, 1, 2.0) == 50.0


ALL_WORKLOADS = ["small-1k", "llama7b-8k", "llama7b-16k", "varlen-10k", "llama13b-32k",
                 "lmhead-llama7b-16k", "attn-llama7b-16k", "predict-llama13b-32k",
                 "mlp-llama7b-16k"]


def test_every_workload_has_its_definition_and_stored_thresholds():
    """Each bench workload names a generator configuration; the layer
    workloads also have their oracle-only stored thresholds."""
    import os

    import bench
    from contextual_token_sparsity_b200 import synth
    here = os.path.dirname(os.path.abspath(__file__))
    for w in ALL_WORKLOADS:
        if w in synth.WORKLOADS:
            if w != "small-1k":  # small enough to score in the tests themselves
                assert os.path.exists(os.path.join(here, "golden", f"{w}.json")), w
                assert bench.thresholds(w, synth.WORKLOADS[w].layers) is not None, w
        elif w.startswith("lmhead-"):
            assert w in synth.LM_HEAD_WORKLOADS, w
        else:  # extension workloads run on a layer workload's shapes
            assert w.split("-", 1)[1] in synth.WORKLOADS, w


@pytest.mark.parametrize("workload", ALL_WORKLOADS)
def test_reference_arm_other_ranks_exit_without_work(workload, monkeypatch, capsys):
    """Under torchrun the reference arm runs on rank 0 only: any other rank
    prints nothing and returns at once (no oracle work, no collective)."""
    import time

    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    t0 = time.perf_counter()
    bench.main(["--impl", "reference", "--gpus", "2", "--workload", workload, "--steps", "1",
                "--warmup", "3"])
    assert time.perf_counter() - t0 < 5.0
    assert capsys.readouterr().out == ""


def test_clock_summary_reports_load_clocks_and_reasons():
    """The clock record of a bench line: median SM clock, the maximum, power
    and every throttle reason seen in any sample (nvidia-smi rows parsed)."""
    import bench
    rows = [["1965", "1965", "410.0", "0x0", "Not Active", "Not Active", "Not Active", "Not Active"],
            ["1500", "1965", "990.5", "0x4", "Not Active", "Not Active", "Not Active", "Active"],
            ["1450", "1965", "995.0", "0x4", "Not Active", "Not Active", "Not Active", "Active"]]
    s = bench.ClockSampler.summary([bench.ClockSampler.parse_smi(r) for r in rows], "nvidia-smi")
    assert s["sm_mhz"] == 1500 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["power_w_max"] == 995.0 and s["reasons"] == ["sw_power_cap"]
    assert bench.ClockSampler.summary([], "nvml") is None


def test_scorer_traffic_record_is_tied_to_the_scorer_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu record only while that
    record was taken on the current scorer source and on the bench workload;
    any other workload, a stale digest, a malformed or a missing file give
    null."""
    import json

    import bench
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("llama7b-16k") is None            # no record
    src = tmp_path / "contextual_token_sparsity_b200" / "csrc"
    src.mkdir(parents=True)
    for name in bench.SCORE_SOURCES:
        (src / name).write_text("// " + name)
    digest = bench.score_source_digest()
    rec = prof / "score_tiles_traffic.json"
    rec.write_text(json.dumps({"workload": "llama7b-16k", "source_digest": digest,
                               "dram_bytes_per_launch": 476498261}))
    assert bench.profiled_traffic("llama7b-16k") == 476498261
    assert bench.profiled_traffic("llama7b-8k") is None              # other workload
    rec.write_text("{not json")
    assert bench.profiled_traffic("llama7b-16k") is None            # malformed
    rec.write_text(json.dumps({"workload": "llama7b-16k", "source_digest": digest,
                               "dram_bytes_per_launch": 476498261}))
    (src / bench.SCORE_SOURCES[0]).write_text("// changed")
    assert bench.profiled_traffic("llama7b-16k") is None            # source changed since


"""The bench's multi-rank plumbing on CPU: two gloo ranks (no GPU).  The timed region's
whole-job time is the maximum over ranks and the throughput counts every rank's tokens;
the reference arm (the oracle on host cores) runs on rank 0 only."""
import importlib.util
import io
import os
import socket
import sys
import contextlib

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _bench()
        ms_local = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms_max, value = bench.job_throughput(ms_local, world, 4096, 3, "cpu")
        out[rank] = (ms_max, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_job_throughput_is_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        ms_max, value = res[r]
        assert ms_max == 15.0  # the slowest rank's time, seen by every rank
        assert value == pytest.approx(world * 4096 * 3 / (15.0 / 1e3))


def test_job_throughput_single_rank_needs_no_process_group():
    bench = _bench()
    ms_max, value = bench.job_throughput(2.5, 1, 1000, 4, "cpu")
    assert ms_max == 2.5 and value == pytest.approx(1000 * 4 / 2.5e-3)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    """Under torchrun only rank 0 times the oracle and prints; other ranks exit without work."""
    bench = _bench()
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "1",
                                      "--steps", "1"])
    args = bench.parse()
    from dropless_mixture_experts_dmoe_b200.workloads import WORKLOADS

    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, WORKLOADS[1])
    assert buf.getvalue() == ""


def test_reference_arm_json_line(monkeypatch):
    """On rank 0 the reference arm prints one JSON line with the contract's keys: the oracle's
    tokens/s as value, cpu_baseline describing the run, and an e2e with no transfers."""
    import json

    bench = _bench()
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "1",
                                      "--steps", "2"])
    args = bench.parse()
    from dropless_mixture_experts_dmoe_b200.workloads import WORKLOADS

    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, WORKLOADS[1])
    lines = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["steps"] == 2
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["T"] == 256 and d["config"]["num_experts"] == 8

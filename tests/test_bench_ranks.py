"""Multi-rank plumbing of bench.py on CPU: two gloo ranks (the GPU runs use one
process per GPU over NCCL with the same calls). Each rank times its own replica of
the workload; the job's time is the slowest rank's, and the whole-job throughput
counts every rank's steps."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        # Rank r reports (r + 1) * 3 ms: the job time is the largest, 3 * world ms.
        ms = bench.max_over_ranks(3.0 * (rank + 1), dist)
        out[rank] = (ms, bench.whole_job_tflops(2e12, 10, world, ms))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_aggregate(world):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(60)
        assert all(p.exitcode == 0 for p in procs)
        res = dict(out)
    assert sorted(res) == list(range(world))
    for ms, tf in res.values():
        assert ms == 3.0 * world
        # world replicas x 10 steps x 2e12 FLOP in 6 ms
        assert tf == pytest.approx(2e12 * 10 * world / 6e-3 / 1e12)


def test_single_process_passthrough():
    assert bench.max_over_ranks(1.25, None) == 1.25
    assert bench.whole_job_tflops(1e12, 4, 1, 2.0) == pytest.approx(2000.0)


def test_call_stats_median_min_max():
    assert bench.call_stats([3.0, 1.0, 2.0]) == {"median": 2.0, "min": 1.0, "max": 3.0, "calls": 3}
    assert bench.call_stats([4.0, 1.0, 2.0, 3.0]) == {"median": 2.5, "min": 1.0, "max": 4.0, "calls": 4}


def test_reference_arm_json_line():
    """`bench.py --impl reference` (the CPU oracle on bounded samples) prints one JSON line
    with the contract's keys; a rank other than 0 prints nothing and exits 0."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3 and d["value"] > 0
    assert d["config"]["workload"] == "square_bf16_4096"
    assert {"value", "unit", "cores", "kind", "sample"} <= set(d["cpu_baseline"])
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=root, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_gpus_n_without_enough_gpus_refuses():
    """`bench.py --gpus 2` started without a launcher starts its own ranks, one per GPU;
    with fewer GPUs visible than asked for it exits with status 2 and times nothing
    (it never reports fewer GPUs than requested)."""
    import subprocess
    import sys
    import torch
    if torch.cuda.device_count() >= 2:
        pytest.skip("two GPUs are visible: the launch would run")
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, bench.__file__, "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 2
    assert "GPU(s) visible" in r.stderr and r.stdout.strip() == ""


def test_world_size_must_match_gpus():
    import subprocess
    import sys
    env = dict(os.environ, WORLD_SIZE="3", RANK="0")
    r = subprocess.run([sys.executable, bench.__file__, "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 2 and "WORLD_SIZE=3" in r.stderr

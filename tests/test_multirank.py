"""The bench's multi-rank host logic on CPU: two gloo ranks.  Every rank runs
an independent replica (weak scaling); the job's times are the maximum over
ranks, taken by one collective that every rank enters; only rank 0 prints;
the reference arm runs on rank 0 alone."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r: step 1.0 + r ms, phases (5 - r, 2 r): the job sees the slowest of each
        red = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 2.0 * rank], dist, "cpu")
        e2e = bench.max_over_ranks([3.0 * (rank + 1)], dist, "cpu")[0]
        with open(os.path.join(out_dir, "r%d.txt" % rank), "w") as f:
            f.write(" ".join(repr(v) for v in red + [e2e]))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        vals = [float(v) for v in open(tmp_path / ("r%d.txt" % r)).read().split()]
        assert vals == [2.0, 5.0, 2.0, 6.0]


def test_single_rank_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]


def test_weak_scaling_job_throughput():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks of 1e12 flop each in 1 ms (the slowest rank) = 2000 TFLOP/s
    assert bench.job_tflops(2, 1e12, 1.0) == pytest.approx(2000.0)
    assert bench.job_tflops(1, 1e12, 2.0) == pytest.approx(500.0)


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the reference arm's other ranks exit 0 without work or output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_json_line():
    """Single rank: one JSON line with the contract's keys; the oracle timed on
    the host as the reference arm."""
    import json
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-500:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["warmup"] >= 3 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0

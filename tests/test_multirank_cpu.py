"""The multi-rank path of the benchmark on CPU (gloo, two ranks): each rank's shard seed,
the max-over-ranks device time and the whole-job throughput, and the reference arm under
torchrun (rank 0 alone prints one line)."""
import json
import os
import socket
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                    # rank 1 is the slower one
        mx = bench.max_over_ranks(ms, world)
        out[rank] = (bench.shard_seed(3, rank), mx, bench.job_throughput(1000, world, 4, mx))
    finally:
        dist.destroy_process_group()


def test_two_rank_time_and_throughput():
    import torch.multiprocessing as mp

    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    seeds = {r: res[r][0] for r in range(world)}
    assert seeds[0] == 3 and seeds[1] != seeds[0]            # each rank its own shard
    for r in range(world):
        assert res[r][1] == 15.0                              # the slowest rank's time on every rank
        assert res[r][2] == pytest.approx(1000 * 2 * 4 / 0.015)


def test_one_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.job_throughput(16384, 1, 10, 2.0) == pytest.approx(16384 * 10 / 0.002)


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--config", "c1_fp32_lowrank"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["cpu_baseline"]["kind"] == "oracle"

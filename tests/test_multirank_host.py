"""The N > 1 path of bench.py on the CPU (gloo, world size 2; no GPU).

bench.py runs one independent replica of the workload per rank (the method has
no exchange step on the replicated path): the job's time is the maximum over
the ranks, its throughput the units of all ranks over that time, and only rank 0
prints.  These tests check the max-over-ranks reduction with two gloo ranks, the
whole-job throughput, and the reference arm under torchrun (rank 0 alone runs
and prints one line; the other rank exits 0 without work)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        ms = [2.5, 3.75][rank]  # rank 1 is the slow replica
        got = bench.reduce_max(ms, world, torch.device("cpu"))
        out[rank] = (got, bench.job_throughput(1000, world, got))
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        got, thr = res[rank]
        assert got == 3.75
        assert thr == pytest.approx(2 * 1000 / 3.75e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.reduce_max(1.25, 1, None) == 1.25
    assert bench.job_throughput(1 << 30, 1, 2.0) == pytest.approx((1 << 30) / 2e-3)


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0

"""The multi-rank host path of bench.py, on the CPU with gloo (world size 2):
barrier and max-over-ranks timing, the weak-scaling aggregate, and the
reference arm under torchrun (rank 0 alone prints, every rank exits 0)."""
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        barrier, max_over_ranks = bench.rank_helpers(torch, dist, torch.device("cpu"))
        barrier()
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        worst = max_over_ranks(local_ms)
        value = bench.weak_scaling_value(world, 2.0e12, worst, 4)
        out[rank] = (worst, value)
        barrier()
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_max_and_weak_scaling():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for worst, value in res.values():
        assert worst == 15.0                  # the slowest rank's time on every rank
        assert value == pytest.approx(2 * 2.0e12 / (15.0 / 4 * 1e-3) / 1e12)


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench
    barrier, max_over_ranks = bench.rank_helpers(torch, None, torch.device("cpu"))
    barrier()
    assert max_over_ranks(3.5) == 3.5
    assert bench.weak_scaling_value(1, 1.0e12, 1000.0, 1) == pytest.approx(1.0)


@pytest.mark.slow
def test_reference_arm_under_torchrun_two_ranks():
    """`bench.py --impl reference` launched as the driver launches it for N = 2:
    rank 0 runs the oracle and prints one JSON line; rank 1 prints nothing."""
    port = _free_port()
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-rows", "2"]
    proc = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [l for l in proc.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, proc.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["cpu_baseline"]["kind"] == "oracle"

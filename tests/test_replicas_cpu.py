"""The multi-GPU path of bench.py (independent replicas, no collective on the data path) on
CPU ranks: gloo, world size 2, rendezvous on 127.0.0.1.  What runs on the GPU per rank is the
single-GPU path the parity tests cover; what is checked here is the host logic around it."""
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
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # the job's time is its slowest rank's, on every rank
        slowest = bench.max_over_ranks(10.0 + 3 * rank, world)
        out[rank] = slowest
        # replicas draw different inputs (seed + rank), so their routing differs
        from routing_dispatch_expert_gemm_b200 import inputs as I
        x, _ = I.make_inputs(I.WORKLOADS["tiny_fp32"], seed=rank, layers=1, experts=False)
        t = x.sum().reshape(1)
        gathered = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(gathered, t)
        out[world + rank] = float(gathered[0] != gathered[1])
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_seeds_gloo():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1] == 13.0
    assert out[2] == out[3] == 1.0


def test_job_throughput_is_weak_scaling():
    # N replicas of T units each, in the slowest rank's step time
    assert bench.job_throughput(1412 * 24, 1, 2.0) == pytest.approx(1412 * 24 / 2e-3)
    assert bench.job_throughput(1412 * 24, 8, 2.0) == pytest.approx(8 * 1412 * 24 / 2e-3)
    assert bench.max_over_ranks(7.5, 1) == 7.5  # a single rank needs no collective


@pytest.mark.slow
def test_reference_arm_under_torchrun_prints_once():
    """--impl reference under torchrun: rank 0 alone runs the oracle and prints one JSON line;
    the other rank exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny_fp32",
           "--steps", "1", "--warmup", "0", "--gpus", "2"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"

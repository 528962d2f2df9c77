"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.

The path has no exchange step (replicas only), so the only cross-rank
operations are the barrier and the max over ranks of the device time.
"""
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


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    bench.dist_barrier(world)
    ms = [3.0, 5.0][rank]                       # rank 1 is the slow one
    m = bench.dist_max(ms, world, device="cpu")
    v = bench.weak_scaling_value(1000, 10, m, world)
    out[rank] = (m, v)
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 5.0
    # 2 ranks x 2 bytes x 1000 weights x 10 steps in 5 ms
    assert res[0][1] == pytest.approx(2 * 2.0 * 1000 * 10 / 5e-3 / 1e9)


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_max(7.0, 1) == 7.0
    assert bench.weak_scaling_value(10, 1, 1.0, 1) == pytest.approx(2 * 10 / 1e-3 / 1e9)


def test_reference_arm_under_torchrun_prints_once():
    """torchrun with 2 ranks: rank 0 alone runs the oracle and prints one JSON line."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "tiny_512", "--reference-budget-s", "2"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    import json
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["e2e"]["h2d_bytes_per_step"] == 0 and d["value"] > 0

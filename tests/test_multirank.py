"""The multi-GPU bench path on CPU: two gloo ranks.

The layer shards by tokens into independent replicas (no exchange step), so
the only collective work in bench.py is the timing reduction: the whole-job
value is (ranks x ops per rank x steps) / (the slowest rank's time).  These
tests run that reduction, and the reference arm's rank handling, across two
processes with the gloo backend.
"""
import json
import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import torch

        import bench

        def reduce_max(x):
            t = torch.tensor([x], dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            return float(t.item())

        value, t_step = bench.aggregate(times[rank], 1e12, world, reduce_max)
        out[rank] = (value, t_step)
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_weak_scaling_value_uses_slowest_rank():
    world = 2
    times = [[0.010, 0.010, 0.010], [0.012, 0.013, 0.011]]  # rank 1 is slower
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), times, out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    slowest = sum(times[1])
    expect = world * 1e12 * 3 / slowest / 1e12
    for rank in range(world):
        value, t_step = res[rank]
        assert value == pytest.approx(expect)          # same on every rank
        assert t_step == pytest.approx(slowest / 3)


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "1"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_on_rank0():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "1", "--workload", "tiny_16x256x256"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0

"""The multi-rank host path of bench.py on CPU: world size 2 over gloo.

Each rank processes its own batch (weak scaling, no data-path collective);
the step time reported is the maximum over ranks and the whole-job value
counts every rank's tokens.  The reference arm runs on rank 0 only.
"""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]
        ms = bench.max_over_ranks(local_ms, torch, dist, device="cpu")
        val = bench.weak_scaling_value(world, 4096, ms)
        out.put((rank, ms, val))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, val in res:
        assert ms == 5.0                       # the slowest rank sets the step time
        assert val == pytest.approx(2 * 4096 / 5e-3)


def test_reference_arm_only_rank0_prints():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_weak_scaling_value_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.weak_scaling_value(1, 16, 0.5) == pytest.approx(32000.0)

"""Multi-rank host paths on CPU over gloo.

bench.py (world size 2): each rank processes its own batch (weak scaling, no
data-path collective); the step time reported is the maximum over ranks and
the whole-job value counts every rank's tokens.  The reference arm runs on
rank 0 only.

Expert parallelism (world sizes 2 and 4): the plan every rank derives from
the all-gathered counts lays out each owner's receive buffer consistently.
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


def _free_port() -> int:
    import socket
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        return s_.getsockname()[1]


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
    port = _free_port()
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


def _ep_plan_worker(rank, world, port, q, E=8):
    import torch
    import torch.distributed as dist
    from sparse_mixture_experts_13_b200.ep import ep_plan_host
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(rank)
        counts = torch.randint(0, 50, (E,), generator=g, dtype=torch.int32)
        if rank == world - 1:
            counts[0] = 0                      # a source with no slots for expert 0
        gathered = [torch.empty(E, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(gathered, counts)
        counts_all = [c.tolist() for c in gathered]
        recv_off, owner_off = ep_plan_host(counts_all, rank, world)
        # share every rank's plan so each owner can check its receive layout
        plans = [None] * world
        dist.all_gather_object(plans, (recv_off, owner_off))
        q.put((rank, counts_all, plans))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,E", [(2, 8), (4, 8), (4, 16)])
def test_ep_plan_gloo(world, E):
    """Expert-parallel plan across gloo ranks: the counts are all-gathered,
    every rank derives the same layout, and in each owner's receive buffer
    the sources' row ranges tile the owner's expert ranges without gap or
    overlap, experts in order and sources in rank order within an expert."""
    ctx = mp.get_context("spawn")
    port = _free_port()
    q = ctx.Queue()
    ps = [ctx.Process(target=_ep_plan_worker, args=(r, world, port, q, E)) for r in range(world)]
    for p_ in ps:
        p_.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p_ in ps:
        p_.join(timeout=60)
        assert p_.exitcode == 0
    res.sort(key=lambda r: r[0])
    counts_all = res[0][1]
    assert all(r[1] == counts_all for r in res)
    plans = res[0][2]
    assert all(r[2] == plans for r in res)
    epr = E // world
    for o in range(world):
        owner_off = plans[o][1]
        assert owner_off[0] == 0
        assert owner_off[epr] == sum(counts_all[r][e] for r in range(world) for e in range(o * epr, (o + 1) * epr))
        for l in range(epr):
            e = o * epr + l
            starts = [plans[r][0][e] for r in range(world)]
            assert starts[0] == owner_off[l]
            for r in range(world - 1):
                assert starts[r + 1] == starts[r] + counts_all[r][e]
            assert starts[-1] + counts_all[world - 1][e] == owner_off[l + 1]

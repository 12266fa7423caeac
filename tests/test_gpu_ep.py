"""Expert parallelism emulated on one GPU: `world` ranks' buffers on one
device, their steps run phase by phase in stream order.  Each rank's output
is compared with the oracle's layer on that rank's tokens; the top-k and
counts bit for bit, y within the layer tolerance."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mixture_experts_13_b200 as moe
    from sparse_mixture_experts_13_b200 import ep
    import gpu_harness as H
else:  # collected on CPU hosts, never run there
    moe = ep = H = None


@pytest.fixture(scope="module")
def o():
    return oracle.Oracle()


def run_ep(o, world, Ts, d, f, E=8, k=2, rows=None, weights=None):
    base = synth.Workload("ep", max(Ts), d, f, E=E, k=k, seed=world)
    if weights is None:
        base.generate()
        weights = (base.W1, base.W3, base.W2)
    else:
        base.generate(weights=False)
    W1, W3, W2 = weights
    xs_host = [synth.normal_bf16(100 + r, synth.TID_X, (T, d)) for r, T in enumerate(Ts)]
    dev_w = [H.to_dev_bf16(W) for W in (W1, W3, W2)]
    Wg = torch.from_numpy(base.Wg).cuda()
    xs = [H.to_dev_bf16(x) for x in xs_host]
    ys, idx, counts = ep.ep_forward_emulated(xs, Wg, *dev_w, world=world, k=k)
    torch.cuda.synchronize()
    for r, T in enumerate(Ts):
        wl = synth.Workload(f"ep{r}", T, d, f, E=E, k=k)
        wl.x, wl.Wg, wl.W1, wl.W3, wl.W2 = xs_host[r], base.Wg, W1, W3, W2
        rt = H.conditional_route(o, wl, idx[r].cpu().numpy(), None, None)
        assert np.array_equal(idx[r].cpu().numpy().reshape(T, k), rt["idx"])
        assert np.array_equal(counts[r].cpu().numpy(), rt["counts"])
        toks = np.arange(T) if rows is None else H.sample_tokens(wl, rt, rows)
        ref = o.layer_rows(wl.x, W1, W3, W2, rt, toks)
        H.assert_close(H.bf16_f64(H.bf16_host(ys[r]))[toks], ref["y"], f"y (rank {r} of {world})")
    return ys


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_ep_small(o, world):
    run_ep(o, world, [97 + 13 * r for r in range(world)], 128, 256)


def test_ep_uneven_and_empty_rank(o):
    """A rank with a single token and expert counts of 16 over 4 ranks."""
    run_ep(o, 4, [1, 300, 64, 129], 128, 192, E=16, k=2)


def test_ep_matches_single_gpu_layer(o):
    """The expert-parallel layer and the single-GPU layer on the same tokens
    agree to bf16 rounding (same routing, same expert arithmetic)."""
    wl = synth.Workload("epsg", 200, 128, 256, seed=4).generate()
    dev = H.Device(wl)
    single = H.bf16_f64(H.run_layer(dev, 1)["y"])
    ys, _, _ = ep.ep_forward_emulated([dev.x[:100], dev.x[100:]], dev.Wg, dev.W1, dev.W3, dev.W2, world=2)
    both = np.concatenate([H.bf16_f64(H.bf16_host(y)) for y in ys])
    assert H.rel_fro(both, single) < 2e-3


def test_ep_mixtral_eight_ranks(o):
    """Mixtral shapes, one expert per rank, 512 tokens per rank (sampled rows)."""
    wl = synth.workload("decode")
    wl.generate()
    run_ep(o, 8, [512] * 8, synth.MIXTRAL_D, synth.MIXTRAL_F, rows=12, weights=(wl.W1, wl.W3, wl.W2))


def test_ep_rejects_capacity_and_bad_world():
    sh = moe.make_shape(16, 128, 256, E=8, k=2, capacity_factor=1.0)
    z = torch.zeros(64, dtype=torch.int32, device="cuda")
    x = torch.zeros(16, 128, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    assert moe.moe_ep_dispatch(sh, 2, x, z, z, z, z, z, ws, ws.numel()) == moe.MOE_ERR_UNSUPPORTED
    sh2 = moe.make_shape(16, 128, 256, E=8, k=2)
    assert moe.moe_ep_dispatch(sh2, 3, x, z, z, z, z, z, ws, ws.numel()) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_ep_plan(z, 8, 2, 2, z, z) == moe.MOE_ERR_INVALID_ARG


def test_ep_layer_one_process_group_of_one(o):
    """The one-process-per-GPU driver (NCCL counts all-gather, receive buffers
    in symmetric memory, barriers) in a group of one rank: its plumbing runs
    end to end on one GPU and matches the oracle."""
    import socket
    import torch.distributed as dist
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        wl = synth.Workload("eplayer", 96, 128, 256, seed=6).generate()
        dev = H.Device(wl)
        layer = ep.EPLayer(dev.Wg, dev.W1, dev.W3, dev.W2, E=wl.E, k=wl.k, max_tokens=wl.T)
        y = layer.forward(dev.x)
        torch.cuda.synchronize()
        r = H.conditional_route(o, wl, H.run_layer(dev, 1)["idx"], None, None)
        ref = o.layer_rows(wl.x, wl.W1, wl.W3, wl.W2, r, np.arange(wl.T))
        H.assert_close(H.bf16_f64(H.bf16_host(y)), ref["y"], "y (EPLayer, one rank)")
        del layer
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,E", [(1, 8), (2, 8), (4, 8), (8, 8), (4, 16), (8, 32)])
def test_ep_plan_kernel_equals_host_plan(world, E):
    """moe_ep_plan (the device plan the layer uses) equals ep_plan_host (the
    host restatement the multi-rank CPU tests check), for every rank, on
    random counts with empty sources and empty experts."""
    from sparse_mixture_experts_13_b200.ep import ep_plan_host
    g = torch.Generator().manual_seed(world * 100 + E)
    counts_all = torch.randint(0, 300, (world, E), generator=g, dtype=torch.int32)
    counts_all[0, 0] = 0
    counts_all[:, E - 1] = 0
    dev_counts = counts_all.cuda().contiguous()
    epr = E // world
    for rank in range(world):
        recv_off = torch.full((E,), -1, dtype=torch.int32, device="cuda")
        owner_off = torch.full((epr + 1,), -1, dtype=torch.int32, device="cuda")
        moe.check(moe.moe_ep_plan(dev_counts, E, rank, world, recv_off, owner_off), "moe_ep_plan")
        want_recv, want_owner = ep_plan_host(counts_all.tolist(), rank, world)
        assert recv_off.cpu().tolist() == want_recv, rank
        assert owner_off.cpu().tolist() == want_owner, rank


def run_ep_capacity(o, world, Ts, d, f, cf, policy, E=8, k=2, seed=11, rows=None, weights=None):
    """Expert parallelism with a capacity, emulated: the ranks' tokens are one
    batch (their concatenation), so the reference is the oracle's layer on
    that batch.  The kept slots must be exactly the oracle's (up to slots
    within the comparison tolerance of an expert's threshold probability),
    and each rank's y must match the oracle's rows for its tokens."""
    T_all = sum(Ts)
    base = synth.Workload("epcap", T_all, d, f, E=E, k=k, capacity_factor=cf, drop_policy=policy, skew=True,
                          seed=seed)
    base.generate(weights=weights is None)
    if weights is not None:
        base.W1, base.W3, base.W2 = weights
    starts = np.concatenate([[0], np.cumsum(Ts)])
    xs = [H.to_dev_bf16(base.x[starts[r]:starts[r + 1]]) for r in range(world)]
    dev_w = [H.to_dev_bf16(W) for W in (base.W1, base.W3, base.W2)]
    info = {}
    ys, idx, counts = ep.ep_forward_emulated(xs, torch.from_numpy(base.Wg).cuda(), *dev_w, world=world, k=k,
                                            capacity_factor=cf, drop_policy=policy, info=info)
    torch.cuda.synchronize()
    epr = info["epr"]
    maps = [m.cpu().numpy() for m in info["row_map"]]
    gpu_idx = np.concatenate([i.cpu().numpy() for i in idx])
    gpu_p = np.concatenate([p.cpu().numpy() for p in info["p"]])
    ret = [r.cpu().numpy() for r in info["ret_row"]]
    kept = np.concatenate([np.array([maps[e // epr][row] >= 0 for e, row in zip(i.cpu().numpy(), rr)], bool)
                           for i, rr in zip(idx, ret)])
    rt = H.conditional_route(o, base, gpu_idx, gpu_p, np.where(kept, 0, -1))
    assert rt["cap"] is not None
    assert np.array_equal(gpu_idx.reshape(T_all, k), rt["idx"])
    assert np.array_equal(kept, rt["slot_pos"] >= 0), "kept slots differ from the oracle's"
    assert (~kept).any(), "the case should drop slots"
    toks = np.arange(T_all) if rows is None else H.sample_tokens(base, rt, rows)
    ref = o.layer_rows(base.x, base.W1, base.W3, base.W2, rt, toks)
    y_all = np.concatenate([H.bf16_f64(H.bf16_host(y)) for y in ys])
    H.assert_close(y_all[toks], ref["y"], f"y (expert parallel, {world} ranks, cf {cf}, policy {policy})")
    fully = np.nonzero((rt["slot_pos"].reshape(T_all, k) < 0).all(1))[0]
    if fully.size:
        assert not y_all[fully].any()
    return rt


@pytest.mark.parametrize("policy", [0, 1], ids=["by_prob", "by_order"])
@pytest.mark.parametrize("cf", [1.0, 1.25])
@pytest.mark.parametrize("world", [2, 8])
def test_ep_capacity(o, world, cf, policy):
    run_ep_capacity(o, world, [61 + 29 * r for r in range(world)], 128, 256, cf, policy)


def test_ep_capacity_uneven_ranks_sixteen_experts(o):
    """Four ranks of 1, 300, 64 and 129 tokens, 16 experts (4 per rank)."""
    for policy in (0, 1):
        run_ep_capacity(o, 4, [1, 300, 64, 129], 128, 192, 1.0, policy, E=16, seed=12)


def test_ep_capacity_mixtral_eight_ranks(o):
    """Mixtral shapes, one expert per rank, skewed routing, cf 1.25."""
    wl = synth.workload("decode")
    wl.generate()
    run_ep_capacity(o, 8, [256] * 8, synth.MIXTRAL_D, synth.MIXTRAL_F, 1.25, 0, rows=12,
                    weights=(wl.W1, wl.W3, wl.W2))


def test_ep_capacity_entry_points_refuse():
    z = torch.zeros(64, dtype=torch.int32, device="cuda")
    x = torch.zeros(16, 128, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    nb = moe.make_shape(16, 128, 256, E=8, k=2, capacity_factor=1.0, drop_policy=moe.MOE_DROP_BY_PROB_NEXT_BEST)
    assert moe.moe_ep_dispatch_cap(nb, 2, 0, z, x, z, z, z, z, z, z, z, ws, ws.numel()) == moe.MOE_ERR_UNSUPPORTED
    assert moe.moe_ep_select(nb, 2, z, z, z, x, x, z, z) == moe.MOE_ERR_UNSUPPORTED
    dl = moe.make_shape(16, 128, 256, E=8, k=2)
    assert moe.moe_ep_dispatch_cap(dl, 2, 0, z, x, z, z, z, z, z, z, z, ws, ws.numel()) == moe.MOE_ERR_INVALID_ARG
    cap = moe.make_shape(16, 128, 256, E=8, k=2, capacity_factor=1.0)
    assert moe.moe_ep_dispatch_cap(cap, 2, 2, z, x, z, z, z, z, z, z, z, ws, ws.numel()) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_ep_dispatch_cap(cap, 2, 0, z, x, z, None, z, z, z, z, z, ws, ws.numel()) == \
        moe.MOE_ERR_INVALID_ARG        # by probability needs the probabilities


def test_ep_layer_capacity_one_process_group_of_one(o):
    """EPLayer with a capacity in a group of one rank: the owner (this rank)
    selects over its slots, which is the single-GPU layer's capacity."""
    import socket
    import torch.distributed as dist
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        for policy in (0, 1):
            wl = synth.Workload("eplcap", 96, 128, 256, seed=6, capacity_factor=1.0, drop_policy=policy,
                                skew=True).generate()
            dev = H.Device(wl)
            layer = ep.EPLayer(dev.Wg, dev.W1, dev.W3, dev.W2, E=wl.E, k=wl.k, max_tokens=wl.T,
                               capacity_factor=wl.capacity_factor, drop_policy=policy)
            y = layer.forward(dev.x)
            torch.cuda.synchronize()
            single = H.bf16_f64(H.run_layer(dev, 1)["y"])
            got = H.bf16_f64(H.bf16_host(y))
            assert H.rel_fro(got, single) < 2e-3, policy       # same routing, same kept slots
            assert np.array_equal(got == 0, single == 0), policy  # the same fully dropped tokens
            del layer
    finally:
        dist.destroy_process_group()

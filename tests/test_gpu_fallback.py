"""The next-best-expert fallback (drop policies 2 and 3) through the C ABI
against the oracle: the layer's top-k and counts bit for bit, y within the
layer tolerance, for the bf16 and the 4-bit experts."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mixture_experts_13_b200 as moe
    import gpu_harness as H
else:  # collected on CPU hosts, never run there
    moe = H = None


@pytest.fixture(scope="module")
def o():
    return oracle.Oracle()


def check_fallback(o, wl, rows=None, q4=False, variants=(0,)):
    dev = H.QDevice(wl, o) if q4 else H.Device(wl)
    gl = H.gpu_logits(dev)
    stats = {}
    for variant in variants:
        lay = H.run_layer_q4(dev, reps=2) if q4 else H.run_layer(dev, variant, reps=2)
        assert np.array_equal(lay["ys"][0], lay["ys"][1])
        r = H.fallback_route(o, wl, lay["idx"], gl, stats)
        assert np.array_equal(lay["idx"].reshape(wl.T, wl.k), r["idx"])
        assert np.array_equal(lay["counts"], r["counts"])
        moved = int(((r["expert"] != r["idx"]) & (r["kept"].reshape(wl.T, wl.k) == 1)).sum())
        assert moved > 0, "the case moves no slot"
        toks = np.arange(wl.T) if rows is None else H.sample_tokens(wl, r, rows)
        if q4:
            ref = o.layer_rows_q4(wl.x, *dev.q_host, r, toks)
        else:
            ref = o.layer_rows(wl.x, wl.W1, wl.W3, wl.W2, r, toks)
        H.assert_close(H.bf16_f64(lay["y"])[toks], ref["y"], f"y (fallback, variant {variant})")
        dropped = np.nonzero((r["kept"].reshape(wl.T, wl.k) == 0).all(1))[0]
        if dropped.size:
            assert not H.bf16_f64(lay["y"])[dropped].any()
    return stats


@pytest.mark.parametrize("policy", [2, 3], ids=["by_prob", "by_order"])
@pytest.mark.parametrize("cf", [0.75, 1.0, 1.25])
def test_fallback_small(o, policy, cf):
    wl = synth.Workload("fb", 256, 128, 448, capacity_factor=cf, drop_policy=policy, skew=True, seed=21).generate()
    check_fallback(o, wl, variants=(1, 2, 3))


@pytest.mark.parametrize("E,k", [(16, 2), (8, 3), (32, 4), (4, 2)])
def test_fallback_expert_counts(o, E, k):
    wl = synth.Workload(f"fbE{E}k{k}", 300, 128, 256, E=E, k=k, capacity_factor=1.0, drop_policy=2, skew=True,
                        seed=E + k).generate()
    check_fallback(o, wl)


def test_fallback_many_slots(o):
    """More than 1024 slots: the look-back grouping over the fallback's experts."""
    wl = synth.Workload("fbmany", 1500, 128, 256, capacity_factor=1.0, drop_policy=3, skew=True, seed=5).generate()
    check_fallback(o, wl)


def test_fallback_q4(o):
    wl = synth.Workload("fbq4", 200, 128, 448, capacity_factor=1.0, drop_policy=2, skew=True, seed=8).generate()
    check_fallback(o, wl, q4=True)


@pytest.mark.parametrize("policy", [2, 3], ids=["by_prob", "by_order"])
def test_fallback_mixtral_skew(o, policy):
    wl = synth.workload("skew")
    wl.generate()
    wl.drop_policy = policy
    check_fallback(o, wl, rows=24)


def test_fallback_stage_permute_unsupported():
    sh = moe.make_shape(64, 128, 448, capacity_factor=1.0, drop_policy=2)
    ws_n = moe.moe_workspace_size(sh)
    ws = torch.empty(ws_n, dtype=torch.uint8, device="cuda")
    t = lambda n, dt=torch.int32: torch.zeros(n, dtype=dt, device="cuda")
    x = torch.zeros(64, 128, dtype=torch.bfloat16, device="cuda")
    st = moe.moe_permute(sh, x, t(128), t(128, torch.float32), t(8), t(9), t(128), t(128),
                         torch.zeros(128, 128, dtype=torch.bfloat16, device="cuda"), ws, ws_n)
    assert st == moe.MOE_ERR_UNSUPPORTED

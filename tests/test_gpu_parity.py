"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Small cases compare every output element; the full Mixtral-shaped cases
(d_model 4096, d_ff 14336, E 8, top-2) compare all routing outputs bit for bit
and a sample of token rows of h, y_perm and y.
"""
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

VARIANTS = [0, 1, 2, 3]
VNAME = {0: "auto", 1: "tiled", 2: "stream", 3: "tiled1"}


@pytest.fixture(scope="module")
def o():
    return oracle.Oracle()


_FULL = {}


def full_workload(name, T=None):
    """Full-size workloads share the seed-0 weights; generate them once."""
    key = (name, T)
    if key not in _FULL:
        wl = synth.workload(name, T=T)
        if "weights" not in _FULL:
            wl.generate(weights=True)
            _FULL["weights"] = (wl.W1, wl.W3, wl.W2)
        else:
            wl.generate(weights=False)
            wl.W1, wl.W3, wl.W2 = _FULL["weights"]
        _FULL[key] = wl
    return _FULL[key]


_DEV = {}


def device_inputs(wl):
    key = id(wl)
    if key not in _DEV:
        if "W" in _DEV and _DEV["W"][0] is wl.W1:
            d = H.Device.__new__(H.Device)
            d.wl = wl
            d.x = H.to_dev_bf16(wl.x)
            d.Wg = torch.from_numpy(wl.Wg).cuda()
            d.W1, d.W3, d.W2 = _DEV["W"][1]
        else:
            d = H.Device(wl)
            if wl.d == synth.MIXTRAL_D:
                _DEV["W"] = (wl.W1, (d.W1, d.W3, d.W2))
        _DEV[key] = d
    return _DEV[key]


def check_everything(o, wl, variant, rows=None, stages=True):
    dev = device_inputs(wl) if wl.d == synth.MIXTRAL_D else H.Device(wl)
    stats = {}
    lay = H.run_layer(dev, variant, reps=2)
    assert np.array_equal(lay["ys"][0], lay["ys"][1]), "layer output not reproducible"
    if stages:
        g = H.run_stages(dev, variant)
        r = H.conditional_route(o, wl, g["idx"].cpu().numpy(), g["p"].cpu().numpy(),
                                g["slot_pos"].cpu().numpy(), stats)
        N = H.compare_routing(g, r, wl)
    else:
        g = None
        r = H.conditional_route(o, wl, lay["idx"], None, None, stats) if wl.capacity_factor <= 0 else None
        assert r is not None
    assert np.array_equal(lay["idx"].reshape(wl.T, wl.k), r["idx"]), "layer topk_idx"
    assert np.array_equal(lay["counts"], r["counts"]), "layer counts"
    toks = np.arange(wl.T) if rows is None else \
        H.sample_tokens(wl, r, rows, block_rows=H.schedule_block_rows(wl.T, variant, wl.k, wl.E))
    ref = o.layer_rows(wl.x, wl.W1, wl.W3, wl.W2, r, toks, want_h=stages, want_o=stages)
    y_gpu = H.bf16_f64(lay["y"])[toks]
    H.assert_close(y_gpu, ref["y"], f"y (layer, {VNAME[variant]})")
    if stages:
        y_st = H.bf16_f64(H.bf16_host(g["y"]))[toks]
        H.assert_close(y_st, ref["y"], f"y (stages, {VNAME[variant]})")
        h_gpu = H.bf16_host(g["h"])
        yp_gpu = H.bf16_host(g["y_perm"])
        hs, hr, os_, or_ = [], [], [], []
        for i, t in enumerate(toks):
            for j in range(wl.k):
                pos = r["slot_pos"][t * wl.k + j]
                if pos < 0:
                    continue
                hs.append(H.bf16_f64(h_gpu[pos]))
                hr.append(ref["h"][i, j])
                os_.append(H.bf16_f64(yp_gpu[pos]))
                or_.append(ref["o"][i, j])
        if hs:
            H.assert_close(np.stack(hs), np.stack(hr), f"h ({VNAME[variant]})")
            H.assert_close(np.stack(os_), np.stack(or_), f"y_perm ({VNAME[variant]})")
        # rows of fully dropped tokens are exactly zero
        dropped = np.nonzero((r["slot_pos"].reshape(wl.T, wl.k) < 0).all(1))[0]
        if dropped.size:
            assert not H.bf16_f64(lay["y"])[dropped].any()
    return stats


# ------------------------------------------------------------------ small cases

@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: VNAME[v])
def test_tiny(o, variant):
    wl = synth.workload("tiny").generate()
    check_everything(o, wl, variant)


@pytest.mark.parametrize("variant", [1, 2, 3], ids=lambda v: VNAME[v])
@pytest.mark.parametrize("policy", [0, 1], ids=["by_prob", "by_order"])
@pytest.mark.parametrize("cf", [0.5, 1.0, 1.25])
def test_tiny_capacity(o, variant, policy, cf):
    wl = synth.Workload("tiny_cap", 256, 128, 448, capacity_factor=cf, drop_policy=policy, skew=True).generate()
    check_everything(o, wl, variant)


@pytest.mark.parametrize("policy", [0, 1], ids=["by_prob", "by_order"])
@pytest.mark.parametrize("cf", [0.75, 1.25])
def test_capacity_many_slots(o, policy, cf):
    """More than 1024 slots take the multi-block look-back grouping."""
    wl = synth.Workload("cap_many", 1000, 128, 256, capacity_factor=cf, drop_policy=policy, skew=True,
                        seed=9).generate()
    check_everything(o, wl, 1)


@pytest.mark.parametrize("E,k", [(4, 1), (16, 2), (8, 3), (32, 4), (8, 8), (1, 1)])
@pytest.mark.parametrize("variant", [1, 2, 3], ids=lambda v: VNAME[v])
def test_expert_counts(o, E, k, variant):
    wl = synth.Workload(f"E{E}k{k}", 96, 128, 256, E=E, k=k, seed=3).generate()
    check_everything(o, wl, variant)


@pytest.mark.parametrize("T", [1, 2, 3, 17, 127, 128, 129, 300])
@pytest.mark.parametrize("variant", [1, 2, 3], ids=lambda v: VNAME[v])
def test_ragged_T(o, T, variant):
    wl = synth.Workload(f"T{T}", T, 192, 320, seed=T).generate()
    check_everything(o, wl, variant)


def test_T_zero_is_noop():
    sh = moe.make_shape(0, 128, 448)
    assert moe.moe_layer_forward(sh, None, None, None, None, None, None, None, None, None, 0) == moe.MOE_OK
    assert moe.moe_router_topk(sh, None, None, None, None, None, None, None) == moe.MOE_OK


@pytest.mark.parametrize("variant", [1, 2, 3], ids=lambda v: VNAME[v])
def test_one_expert_takes_every_token(o, variant):
    """Expert 5 is every token's first choice; several experts stay empty."""
    wl = synth.Workload("hot5", 200, 128, 256, seed=5).generate()
    wl.x[:, 3] = 0x3F80
    wl.Wg[5, 3] += 40.0
    wl.Wg[0, 3] += 20.0        # second choice: mostly expert 0
    check_everything(o, wl, variant)


@pytest.mark.parametrize("variant", [1, 2, 3], ids=lambda v: VNAME[v])
def test_exact_logit_ties(o, variant):
    """Experts 2 and 3 have identical router rows, so their logits tie
    exactly; the smaller index must win, as in the oracle."""
    wl = synth.Workload("ties", 64, 128, 256, seed=8).generate()
    wl.Wg[3] = wl.Wg[2]
    wl.Wg[2] += 3.0 * np.abs(wl.Wg[2]).max()  # make 2/3 the top pair for many tokens
    wl.Wg[3] = wl.Wg[2]
    dev = H.Device(wl)
    g = H.run_stages(dev, variant)
    idx = g["idx"].cpu().numpy().reshape(64, 2)
    both = (idx == 2).any(1) & (idx == 3).any(1)
    assert both.any()
    assert np.all(idx[both, 0] == 2) and np.all(idx[both, 1] == 3)
    check_everything(o, wl, variant)


def test_tensor_core_router_ties(o):
    """1100 tokens at d=512 take the tensor-core router (T >= 192, d a
    multiple of 512), with a ragged last tile of 12 tokens: experts 2 and 3
    tie exactly for many tokens (the smaller index wins), and zero rows pick
    experts 0 and 1 with gates 1/2, as in the oracle."""
    wl = synth.Workload("ties_mma", 1100, 512, 256, seed=9).generate()
    wl.Wg[2] += 3.0 * np.abs(wl.Wg[2]).max()
    wl.Wg[3] = wl.Wg[2]
    wl.x[:10] = 0
    g = H.run_stages(H.Device(wl), 1)
    idx = g["idx"].cpu().numpy().reshape(1100, 2)
    both = (idx == 2).any(1) & (idx == 3).any(1)
    assert both.sum() > 100
    assert np.all(idx[both, 0] == 2) and np.all(idx[both, 1] == 3)
    assert np.all(idx[:10] == [0, 1]) and np.all(g["w"].cpu().numpy().reshape(1100, 2)[:10] == 0.5)
    check_everything(o, wl, 1)


def test_zero_input_ties():
    """x = 0: all logits are 0, the experts 0..k-1 are chosen, gates are 1/k
    and the output is exactly zero."""
    wl = synth.Workload("zeros", 40, 128, 256).generate()
    wl.x[:] = 0
    for variant in (1, 2, 3):
        g = H.run_stages(H.Device(wl), variant)
        assert np.all(g["idx"].cpu().numpy().reshape(40, 2) == [0, 1])
        assert np.all(g["w"].cpu().numpy() == 0.5)
        assert not H.bf16_host(g["y"]).any()


def test_capacity_zero_and_huge(o):
    wl = synth.Workload("cap0", 4, 128, 256, capacity_factor=0.5).generate()   # cap = 0
    for variant in (1, 2, 3):
        lay = H.run_layer(H.Device(wl), variant)
        assert not lay["y"].any()
    base = synth.Workload("nocap", 100, 128, 256, seed=2).generate()
    huge = synth.Workload("hugecap", 100, 128, 256, seed=2, capacity_factor=1e9).generate()
    for variant in (1, 2, 3):
        a = H.run_layer(H.Device(base), variant)["y"]
        b = H.run_layer(H.Device(huge), variant)["y"]
        assert np.array_equal(a, b)


def test_variants_agree_closely():
    """Both schedules compute the same function (rounding differs only in
    the order of fp32 accumulation)."""
    wl = synth.Workload("v", 100, 256, 512, seed=11).generate()
    a = H.bf16_f64(H.run_layer(H.Device(wl), 1)["y"])
    for v in (2, 3):
        b = H.bf16_f64(H.run_layer(H.Device(wl), v)["y"])
        assert H.rel_fro(a, b) < 5e-3


# ------------------------------------------------------- Mixtral-shaped sizes

@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: VNAME[v])
def test_decode_T16(o, variant):
    check_everything(o, full_workload("decode"), variant, rows=16)


@pytest.mark.parametrize("variant", [0, 2, 3], ids=lambda v: VNAME[v])
def test_prefill_T4096(o, variant):
    check_everything(o, full_workload("prefill"), variant, rows=64)


@pytest.mark.parametrize("policy", [0, 1], ids=["by_prob", "by_order"])
def test_skew_T8192_capacity(o, policy):
    wl = full_workload("skew")
    wl.drop_policy = policy
    stats = check_everything(o, wl, 0, rows=64)
    share = float((H.run_layer(device_inputs(wl), 0)["counts"][0])) / (wl.T * wl.k)
    assert 0.37 < share < 0.43, share
    wl.drop_policy = 0


@pytest.mark.parametrize("E,d,T,k", [(5, 1024, 2051, 2), (8, 2048, 1024, 2), (2, 4096, 1031, 2), (1, 512, 1030, 1),
                                     (8, 1024, 1100, 3), (8, 512, 192, 2), (6, 1024, 777, 2)])
def test_tensor_core_router_shapes(o, E, d, T, k):
    """The tensor-core router (from 192 tokens) with fewer than 8 experts
    (unused MMA columns, down to a single expert), top-1 and top-3, a
    quarter of d per CTA of 1 to 8 MMA steps per warp, and tiles that the
    clusters share unevenly (or one tile per cluster), the last one ragged;
    every row is compared."""
    wl = synth.Workload(f"mma_router{E}_{d}_{k}", T, d, 128, E=E, k=k, seed=E + d + k).generate()
    check_everything(o, wl, 1)


@pytest.mark.parametrize("T", [1, 8, 64, 512, 32768])
def test_sweep(o, T):
    check_everything(o, full_workload("sweep", T=T), 0, rows=64 if T >= 4096 else 16)


def test_gate_up_split_along_k(o):
    """Two Mixtral tokens: the streaming gate/up GEMM is split 2 ways along K
    (fp32 partials, then their sum through SiLU * mul); T = 1 in the sweep
    takes the same path."""
    check_everything(o, full_workload("sweep", T=2), 0, rows=16)


@pytest.mark.parametrize("E", [8, 16, 32])
def test_router_many_tokens(o, E):
    """700 tokens at d=128: the register router for E=8, the grouped router
    with several tokens per block for E=16 and 32."""
    wl = synth.Workload(f"many{E}", 700, 128, 192, E=E, k=2, seed=E).generate()
    check_everything(o, wl, 1)

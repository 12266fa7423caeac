"""Parity of the 4-bit expert path (through the C ABI) with the CPU oracle.

The quantiser is compared byte for byte with the oracle's; the layer and the
grouped GEMMs consume the oracle's codes and scales and are compared with
the oracle's 4-bit layer under the same rules as the bf16 path (routing bit
for bit; h, y_perm and y by relative Frobenius error <= 5e-3 and per element
<= 2e-2 of the largest reference value).
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


@pytest.fixture(scope="module")
def o():
    return oracle.Oracle()


def gpu_quantize(W: np.ndarray):
    E, R, K = W.shape
    Wd = H.to_dev_bf16(W)
    codes = torch.empty(E, R, K // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(E, K // 64, R, dtype=torch.bfloat16, device="cuda")
    moe.check(moe.moe_quantize_q4(Wd, E, R, K, codes, scales), "quantize_q4")
    torch.cuda.synchronize()
    return codes.cpu().numpy(), H.bf16_host(scales)


def awkward_matrix(rng, E, R, K):
    """Random weights plus blocks that stress the rounding: all zero, exact
    half steps (w / s = n + 1/2, ties to even), a lone large value, tiny
    magnitudes near the bf16 subnormal range."""
    W = rng.standard_normal((E, R, K)).astype(np.float32)
    W[0, 0, :64] = 0.0
    steps = np.array([3.5, -2.5, 0.5, -0.5, 1.5, 6.5, -6.5, 7.0], np.float32)
    W[0, 1, -64:] = np.resize(steps, 64) * np.float32(2.0 ** -3)
    W[0, 2, :64] = 1e-3
    W[0, 2, 5] = 50.0
    W[-1, -1, -64:] = rng.standard_normal(64).astype(np.float32) * np.float32(1e-36)
    return synth.f32_to_bf16(W)


@pytest.mark.parametrize("E,R,K", [(1, 8, 64), (3, 200, 192), (2, 64, 4160)])
def test_quantizer_bit_exact(o, E, R, K):
    W = awkward_matrix(np.random.default_rng(E * R + K), E, R, K)
    c_ref, s_ref = o.q4_quantize(W)
    c, s = gpu_quantize(W)
    assert np.array_equal(s, s_ref), "scales"
    assert np.array_equal(c, c_ref), "codes"


def test_quantizer_full_expert_matrix(o):
    """One Mixtral-sized expert matrix [1, 14336, 4096] byte for byte."""
    wl = synth.Workload("q", 1, 4096, 14336, E=1)
    wl.generate()
    c_ref, s_ref = o.q4_quantize(wl.W1)
    c, s = gpu_quantize(wl.W1)
    assert np.array_equal(s, s_ref) and np.array_equal(c, c_ref)


def test_quantizer_rejects_bad_sizes():
    W = torch.zeros(2, 64, 128, dtype=torch.bfloat16, device="cuda")
    c = torch.empty(2, 64, 64, dtype=torch.uint8, device="cuda")
    s = torch.empty(2, 2, 64, dtype=torch.bfloat16, device="cuda")
    E = moe.MOE_ERR_INVALID_ARG
    assert moe.moe_quantize_q4(W, 2, 64, 96, c, s) == E     # K % 64
    assert moe.moe_quantize_q4(W, 2, 60, 128, c, s) == E    # R % 8
    assert moe.moe_quantize_q4(W, 0, 64, 128, c, s) == E
    assert moe.moe_quantize_q4(None, 2, 64, 128, c, s) == E


def check_q4(o, wl, rows=None, stages=True, q=None):
    dev = H.QDevice(wl, o, q)
    lay = H.run_layer_q4(dev, reps=2)
    assert np.array_equal(lay["ys"][0], lay["ys"][1]), "layer output not reproducible"
    stats = {}
    if stages:
        g = H.run_stages_q4(dev)
        r = H.conditional_route(o, wl, g["idx"].cpu().numpy(), g["p"].cpu().numpy(), g["slot_pos"].cpu().numpy(),
                                stats)
        H.compare_routing(g, r, wl)
    else:
        assert wl.capacity_factor <= 0
        r = H.conditional_route(o, wl, lay["idx"], None, None, stats)
    assert np.array_equal(lay["idx"].reshape(wl.T, wl.k), r["idx"]), "layer topk_idx"
    assert np.array_equal(lay["counts"], r["counts"]), "layer counts"
    toks = np.arange(wl.T) if rows is None else H.sample_tokens(wl, r, rows)
    ref = o.layer_rows_q4(wl.x, *dev.q_host, r, toks, want_h=stages, want_o=stages)
    H.assert_close(H.bf16_f64(lay["y"])[toks], ref["y"], "y (q4 layer)")
    if stages:
        H.assert_close(H.bf16_f64(H.bf16_host(g["y"]))[toks], ref["y"], "y (q4 stages)")
        h_gpu, yp_gpu = H.bf16_host(g["h"]), H.bf16_host(g["y_perm"])
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
            H.assert_close(np.stack(hs), np.stack(hr), "h (q4)")
            H.assert_close(np.stack(os_), np.stack(or_), "y_perm (q4)")
        dropped = np.nonzero((r["slot_pos"].reshape(wl.T, wl.k) < 0).all(1))[0]
        if dropped.size:
            assert not H.bf16_f64(lay["y"])[dropped].any()
    return dev


def test_q4_tiny(o):
    check_q4(o, synth.workload("tiny").generate())


@pytest.mark.parametrize("T", [1, 2, 17, 33, 65, 129, 300])
def test_q4_ragged_T(o, T):
    """Token tiles of 16, 32, 64 and 128 with a ragged last tile."""
    check_q4(o, synth.Workload(f"q4T{T}", T, 192, 320, seed=T).generate())


@pytest.mark.parametrize("d,f", [(64, 64), (192, 4160), (4160, 192)])
def test_q4_half_stage_K(o, d, f):
    """K = 64 (mod 128): the last 128-input stage is half out of range."""
    check_q4(o, synth.Workload(f"q4d{d}f{f}", 20, d, f, seed=d + f).generate())


@pytest.mark.parametrize("E,k", [(4, 1), (16, 2), (32, 4), (8, 8), (1, 1)])
def test_q4_expert_counts(o, E, k):
    check_q4(o, synth.Workload(f"q4E{E}k{k}", 96, 128, 256, E=E, k=k, seed=3).generate())


@pytest.mark.parametrize("policy", [0, 1], ids=["by_prob", "by_order"])
@pytest.mark.parametrize("cf", [0.5, 1.25])
def test_q4_capacity(o, policy, cf):
    wl = synth.Workload("q4cap", 256, 128, 448, capacity_factor=cf, drop_policy=policy, skew=True).generate()
    check_q4(o, wl)


_FULL = {}


def full_q4(o, T):
    """Mixtral-sized workload (seed 0 weights) with its oracle codes."""
    if "w" not in _FULL:
        wl = synth.workload("decode")
        wl.generate(weights=True)
        _FULL["w"] = (wl.W1, wl.W3, wl.W2)
        _FULL["q"] = tuple(o.q4_quantize(W) for W in _FULL["w"])
    wl = synth.workload("sweep", T=T) if T != 16 else synth.workload("decode")
    wl.generate(weights=False)
    wl.W1, wl.W3, wl.W2 = _FULL["w"]
    return wl, _FULL["q"]


@pytest.mark.parametrize("T", [16, 1, 32, 64, 72, 512])
def test_q4_mixtral_sizes(o, T):
    """Integer-MMA kernels at T = 1, 16, 32 and 64 (16-token tiles,
    256-input stages; at 64 some experts spill into a second tile) and 72
    (32-token tiles, 128-input stages); the dequantising kernels at 512."""
    wl, q = full_q4(o, T)
    check_q4(o, wl, rows=16, q=q)


def test_q4_close_to_bf16_layer(o):
    """The 4-bit layer stays within the quantisation error of the bf16 layer
    (the same weights before quantisation): relative Frobenius < 0.2 for
    N(0, 1/d) weights (4-bit steps of about absmax/7)."""
    wl = synth.Workload("q4vsbf16", 64, 256, 512, seed=5).generate()
    yq = H.bf16_f64(H.run_layer_q4(H.QDevice(wl, o))["y"])
    yb = H.bf16_f64(H.run_layer(H.Device(wl), 2)["y"])
    assert H.rel_fro(yq, yb) < 0.2

"""The whole-layer entry points other than moe_layer_forward, on the GPU.

* moe_layer_forward_host takes x and y in host memory and queues the two
  copies and the layer: the call of a caller whose activations live on the
  host, and the one the end-to-end figure of the benchmark times.  From 4096
  dropless tokens on it runs the layer on groups of tokens whose copies
  overlap the other groups' kernels (the "chunked" case).
* moe_layer_forward_profiled and moe_layer_forward_q4_profiled record six
  CUDA events between the kernels: the benchmark's per-kernel timings.

Each launches the kernels of moe_layer_forward (or moe_layer_forward_q4) with
the same workspace layout, so its y must equal that entry point's bit for
bit.  The tiny workload through host buffers is also compared with the oracle
directly, under the layer's tolerance.
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

CASES = {
    "tiny": dict(T=64, d=128, f=448),                                              # streaming schedule
    "ragged": dict(T=300, d=256, f=512, seed=3),                                   # CTA pairs, ragged tiles
    "cap_by_prob": dict(T=256, d=128, f=256, capacity_factor=1.0, skew=True),      # capacity select kernel
    "next_best": dict(T=256, d=128, f=256, capacity_factor=1.0, drop_policy=2, skew=True),  # fallback kernels
    "chunked": dict(T=6000, d=128, f=256, seed=4),  # host buffers in 2 groups of 3000 tokens, copies overlapped
}


def _device(name):
    return H.Device(synth.Workload(name, **CASES[name]).generate())


def _pinned_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


def _host_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).numpy().view(np.uint16).copy()


@pytest.mark.parametrize("name", list(CASES))
def test_host_buffers_equal_device_entry_point(name):
    """Two calls in a row on a side stream with different x: each y equals
    moe_layer_forward's for that x (the staged x of the first call must not
    leak into the second)."""
    dev = _device(name)
    wl = dev.wl
    sh = dev.shape()
    n = moe.moe_workspace_size(sh)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    xs = [wl.x, synth.normal_bf16(wl.seed + 100, synth.TID_X, (wl.T, wl.d))]
    for call, x_bits in enumerate(xs):
        dev.x = H.to_dev_bf16(x_bits)
        ref = H.run_layer(dev)["y"]
        x_host = _pinned_bf16(x_bits)
        y_host = torch.full((wl.T, wl.d), float("nan"), dtype=torch.bfloat16).pin_memory()
        moe.check(moe.moe_layer_forward_host(sh, x_host, dev.Wg, dev.W1, dev.W3, dev.W2, y_host, ws, n, s),
                  "moe_layer_forward_host")
        assert moe.moe_read_device_status(ws, s) == moe.MOE_OK
        assert np.array_equal(_host_bits(y_host), ref), (name, call)


def test_host_buffers_tiny_against_oracle():
    dev = _device("tiny")
    wl = dev.wl
    sh = dev.shape()
    n = moe.moe_workspace_size(sh)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    y_host = torch.empty((wl.T, wl.d), dtype=torch.bfloat16).pin_memory()
    moe.check(moe.moe_layer_forward_host(sh, _pinned_bf16(wl.x), dev.Wg, dev.W1, dev.W3, dev.W2, y_host, ws, n),
              "moe_layer_forward_host")
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    ref = oracle.Oracle().layer(wl.x, wl.Wg, wl.W1, wl.W3, wl.W2, wl.k)["y"]
    H.assert_close(H.bf16_f64(_host_bits(y_host)), ref, "y (host buffers)")


def _check_clock_records(ws):
    """The two expert GEMMs' {cycles, ns} records at entry and exit (bytes
    64 .. 127 of the workspace) give a plausible SM clock."""
    rec = ws[64:128].view(torch.int64).cpu().numpy()
    for g in (0, 4):
        c0, n0, c1, n1 = (int(v) for v in rec[g:g + 4])
        assert c1 > c0 and n1 > n0, rec
        mhz = (c1 - c0) / (n1 - n0) * 1e3
        assert 300.0 < mhz < 3000.0, mhz


def _check_events(evs):
    torch.cuda.synchronize()
    gaps = [evs[i].elapsed_time(evs[i + 1]) for i in range(5)]
    total = evs[0].elapsed_time(evs[5])
    assert all(g >= 0.0 for g in gaps), gaps
    assert total > 0.0 and abs(sum(gaps) - total) <= 1e-3, (gaps, total)


@pytest.mark.parametrize("variant", [1, 2, 3], ids=["tiled", "stream", "tiled1"])
@pytest.mark.parametrize("name", ["ragged", "cap_by_prob", "next_best"])
def test_profiled_equals_layer(name, variant):
    dev = _device(name)
    wl = dev.wl
    ref = H.run_layer(dev, variant)["y"]
    sh = dev.shape(variant)
    n = moe.moe_workspace_size(sh)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    moe.check(moe.moe_layer_forward_profiled(sh, dev.x, dev.Wg, dev.W1, dev.W3, dev.W2, y, evs, ws, n),
              "moe_layer_forward_profiled")
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    assert np.array_equal(H.bf16_host(y), ref), (name, variant)
    _check_events(evs)
    _check_clock_records(ws)


@pytest.mark.parametrize("name", ["tiny", "cap_by_prob"])
def test_q4_profiled_equals_q4_layer(name):
    wl = synth.Workload(name, **CASES[name]).generate()
    dev = H.QDevice(wl, oracle.Oracle())
    ref = H.run_layer_q4(dev)["y"]
    sh = dev.shape(0)
    n = moe.moe_workspace_size_q4(sh)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    moe.check(moe.moe_layer_forward_q4_profiled(sh, dev.x, dev.Wg, *dev.q, y, evs, ws, n),
              "moe_layer_forward_q4_profiled")
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    assert np.array_equal(H.bf16_host(y), ref), name
    _check_events(evs)
    _check_clock_records(ws)


@pytest.mark.parametrize("name", ["tiny", "cap_by_prob"])
def test_q4_host_buffers_equal_q4_layer(name):
    """moe_layer_forward_q4_host (x and y in page-locked host memory) gives
    moe_layer_forward_q4's output bit for bit, on two calls in a row with
    different tokens on a side stream."""
    wl = synth.Workload(name, **CASES[name]).generate()
    dev = H.QDevice(wl, oracle.Oracle())
    sh = dev.shape(0)
    n = moe.moe_workspace_size_q4(sh)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    for call, x_bits in enumerate([wl.x, synth.normal_bf16(wl.seed + 100, synth.TID_X, (wl.T, wl.d))]):
        dev.x = H.to_dev_bf16(x_bits)
        ref = H.run_layer_q4(dev)["y"]
        y_host = torch.full((wl.T, wl.d), float("nan"), dtype=torch.bfloat16).pin_memory()
        moe.check(moe.moe_layer_forward_q4_host(sh, _pinned_bf16(x_bits), dev.Wg, *dev.q, y_host, ws, n, s),
                  "moe_layer_forward_q4_host")
        assert moe.moe_read_device_status(ws, s) == moe.MOE_OK
        assert np.array_equal(_host_bits(y_host), ref), (name, call)

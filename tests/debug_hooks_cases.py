"""GPU cases for the debug build only (libmoe_debug.so).  Not collected by a
plain `pytest tests`: test_gpu_debug_build.py runs this file, with
MOE_LIB=debug, in a child process.

* The stage-failure hook: MOE_DEBUG_FAIL_STAGE=n makes moe_layer_forward
  return MOE_ERR_CUDA just before queuing stage n, so nothing from stage n
  on runs: y and the exported indices keep their sentinels, and the router's
  histogram in the workspace shows whether stage 1 ran.
* Device-side bounds checks: offsets past the T * k rows handed to
  moe_grouped_swiglu, and an expert index >= E handed to moe_permute, are
  refused by the kernels (MOE_ERR_BOUNDS in the status word) with every
  access kept inside the buffers.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

import sparse_mixture_experts_13_b200 as moe  # noqa: E402
import gpu_harness as H  # noqa: E402

SENTINEL = 0x7FC1  # a NaN bit pattern no layer output has
COUNTS_OFFSET = 256  # counts [E] int32 follow the 16-byte header, 256-byte aligned


def setup_module():
    assert moe.moe_debug_build() == 1, "run with MOE_LIB=debug"


@pytest.mark.parametrize("stage", [1, 2, 3, 4, 5])
def test_stage_failure_queues_nothing_after(stage, monkeypatch):
    wl = synth.Workload("fail", 96, 128, 256, seed=3).generate()
    dev = H.Device(wl)
    ref = H.run_layer(dev, 1)
    sh = dev.shape(1)
    nws = moe.moe_workspace_size(sh)
    ws = torch.zeros(nws, dtype=torch.uint8, device="cuda")
    S = wl.T * wl.k
    y = torch.full((wl.T, wl.d), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    idx = torch.full((S,), -7, dtype=torch.int32, device="cuda")
    counts = torch.full((wl.E,), -7, dtype=torch.int32, device="cuda")
    monkeypatch.setenv("MOE_DEBUG_FAIL_STAGE", str(stage))
    st = moe.moe_layer_forward(sh, dev.x, dev.Wg, dev.W1, dev.W3, dev.W2, y, idx, counts, ws, nws)
    assert st == moe.MOE_ERR_CUDA
    torch.cuda.synchronize()
    yb = y.view(torch.int16).cpu().numpy()
    if stage <= 4:
        assert (yb == SENTINEL).all(), "the combine ran"
    else:
        assert np.array_equal(H.bf16_host(y), ref["y"]), "stages 1-4 ran fully"
    assert (idx.cpu().numpy() == -7).all() and (counts.cpu().numpy() == -7).all()
    hist = ws[COUNTS_OFFSET:COUNTS_OFFSET + 4 * wl.E].view(torch.int32).cpu().numpy()
    assert int(hist.sum()) == (0 if stage == 1 else S)
    # the hook off again: the same workspace gives the reference output
    monkeypatch.delenv("MOE_DEBUG_FAIL_STAGE")
    moe.check(moe.moe_layer_forward(sh, dev.x, dev.Wg, dev.W1, dev.W3, dev.W2, y, idx, counts, ws, nws), "layer")
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    assert np.array_equal(H.bf16_host(y), ref["y"])


@pytest.mark.parametrize("variant", [1, 2, 3], ids=["tiled", "stream", "tiled1"])
def test_offsets_past_the_rows_are_refused(variant):
    wl = synth.Workload("badoff", 40, 128, 256, seed=5).generate()
    dev = H.Device(wl)
    sh = dev.shape(variant)
    S = wl.T * wl.k
    nws = moe.moe_workspace_size(sh)
    ws = torch.zeros(nws, dtype=torch.uint8, device="cuda")
    x_perm = torch.zeros(S, wl.d, dtype=torch.bfloat16, device="cuda")
    h = torch.zeros(S, wl.f, dtype=torch.bfloat16, device="cuda")
    y_perm = torch.zeros(S, wl.d, dtype=torch.bfloat16, device="cuda")
    offsets = torch.tensor(np.linspace(0, S + 64, wl.E + 1).astype(np.int32), device="cuda")
    with H.guarded(sh, ws, nws):
        moe.check(moe.moe_grouped_swiglu(sh, x_perm, offsets, dev.W1, dev.W3, dev.W2, h, y_perm, ws, nws), "gemms")
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_BOUNDS
    assert not H.bf16_host(h).any() and not H.bf16_host(y_perm).any()


@pytest.mark.parametrize("T", [64, 700], ids=["small_path", "lookback_path"])
def test_expert_index_out_of_range_is_refused(T):
    wl = synth.Workload("badidx", T, 128, 256, seed=7).generate()
    dev = H.Device(wl)
    sh = dev.shape(1)
    S = T * wl.k
    nws = moe.moe_workspace_size(sh)
    ws = torch.zeros(nws, dtype=torch.uint8, device="cuda")
    g = H.run_stages(dev, 1)
    idx = g["idx"].clone()
    counts = g["counts"].clone()
    bad = 2 * (T // 3) + 1
    e_bad = int(idx[bad].item())
    idx[bad] = wl.E                      # an expert that does not exist
    counts[e_bad] -= 1                   # the histogram of the valid slots
    out = {n: torch.full((S,), -7, dtype=torch.int32, device="cuda") for n in ("slot_pos", "perm_slot")}
    offsets = torch.empty(wl.E + 1, dtype=torch.int32, device="cuda")
    x_perm = torch.zeros(S, wl.d, dtype=torch.bfloat16, device="cuda")
    with H.guarded(sh, ws, nws):
        moe.check(moe.moe_permute(sh, dev.x, idx, g["p"], counts, offsets, out["slot_pos"], out["perm_slot"], x_perm,
                                  ws, nws), "permute")
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_BOUNDS
    sp = out["slot_pos"].cpu().numpy()
    assert sp[bad] == -1
    ok = np.arange(S) != bad
    ref = g["slot_pos"].cpu().numpy()
    # rows of the valid slots are the reference rows closed up over the refused one
    assert np.array_equal(np.argsort(sp[ok], kind="stable"), np.argsort(ref[ok], kind="stable"))

"""moe_permute_noalloc: the permutation entry point for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).

Through the C ABI, its outputs must equal moe_permute's, bit for bit (they are
integer and copy results), on two calls in a row, so that the contents the
first call leaves in the shared scratch cannot leak into the second.  This
file is collected last on purpose; test_runs_alone_in_a_fresh_process runs
the rest of it again in a new process, where the first call on the device
also does the address look-up.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _route(moe, wl, sh):
    T, E, k = wl.T, wl.E, wl.k
    S = T * k
    x = _dev_bf16(wl.x)
    Wg = torch.from_numpy(wl.Wg).cuda()
    idx = torch.empty(S, dtype=torch.int32, device="cuda")
    w = torch.empty(S, dtype=torch.float32, device="cuda")
    p = torch.empty(S, dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    moe.check(moe.moe_router_topk(sh, x, Wg, None, idx, w, p, counts), "router")
    return x, idx, p, counts


def _outputs(wl):
    S = wl.T * wl.k
    return dict(offsets=torch.full((wl.E + 1,), -7, dtype=torch.int32, device="cuda"),
                slot_pos=torch.full((S,), -7, dtype=torch.int32, device="cuda"),
                perm_slot=torch.full((S,), -7, dtype=torch.int32, device="cuda"),
                x_perm=torch.zeros(S, wl.d, dtype=torch.bfloat16, device="cuda"))


@pytest.mark.parametrize("case", [
    dict(T=300, d=128, f=256, E=8, k=2),                                    # dropless, ragged tiles
    dict(T=256, d=128, f=256, E=8, k=2, capacity_factor=1.0, skew=True),    # capacity, drop by probability
    dict(T=256, d=128, f=256, E=8, k=2, capacity_factor=0.5, drop_policy=1, skew=True),  # by token order
    dict(T=32768, d=64, f=64, E=32, k=2, seed=4),                            # the size limit: 65536 slots
    # more than 1024 slots: the look-back path, with capacity thresholds and drops by rank
    dict(T=4096, d=128, f=256, E=8, k=2, capacity_factor=1.0, skew=True, seed=6),
    dict(T=4096, d=128, f=256, E=8, k=2, capacity_factor=1.0, drop_policy=1, skew=True, seed=6),
], ids=["dropless", "cap_by_prob", "cap_by_order", "max_slots", "lookback_cap_by_prob", "lookback_cap_by_order"])
def test_noalloc_matches_workspace_entry_point(case):
    import sparse_mixture_experts_13_b200 as moe
    wl = synth.Workload("noalloc", **case).generate(weights=False)
    sh = moe.make_shape(wl.T, wl.d, wl.f, wl.E, wl.k, wl.capacity_factor, wl.drop_policy)
    x, idx, p, counts = _route(moe, wl, sh)
    ref = _outputs(wl)
    nws = moe.moe_workspace_size(sh)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    moe.check(moe.moe_permute(sh, x, idx, p, counts, ref["offsets"], ref["slot_pos"], ref["perm_slot"],
                              ref["x_perm"], ws, nws), "moe_permute")
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    N = int(ref["offsets"][-1].item())
    for call in range(2):
        got = _outputs(wl)
        moe.check(moe.moe_permute_noalloc(sh, x, idx, p, counts, got["offsets"], got["slot_pos"],
                                          got["perm_slot"], got["x_perm"]), "moe_permute_noalloc")
        assert moe.moe_permute_noalloc_status() == moe.MOE_OK, call
        assert torch.equal(got["offsets"], ref["offsets"]), call
        assert torch.equal(got["slot_pos"], ref["slot_pos"]), call
        assert torch.equal(got["perm_slot"][:N], ref["perm_slot"][:N]), call
        assert torch.equal(got["x_perm"][:N].view(torch.int16), ref["x_perm"][:N].view(torch.int16)), call


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import sparse_mixture_experts_13_b200 as moe
    sh = moe.make_shape(32769, 64, 64, 8, 2)          # 65538 slots > 65536
    ok = 1 << 20
    assert moe.moe_permute_noalloc(sh, ok, ok, ok, ok, ok, ok, ok, ok) == moe.MOE_ERR_UNSUPPORTED


def test_runs_alone_in_a_fresh_process():
    """The comparisons above, alone in a new process: the first
    moe_permute_noalloc call there does the per-device set-up."""
    here = os.path.abspath(__file__)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", here, "-k",
                        "not fresh_process"], capture_output=True, text=True, timeout=900,
                       cwd=os.path.dirname(os.path.dirname(here)))
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout

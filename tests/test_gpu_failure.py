"""Failure detection on the GPU without a GPU fault.

The bounded device waits (mbarrier phases of the GEMM pipelines, look-back
words of the permutation scan) are made to run out on a barrier and a word
that nothing completes; the kernel must record MOE_ERR_TIMEOUT in the status
word, return normally, and leave the context usable for a correct layer call.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_stays_usable():
    import sparse_mixture_experts_13_b200 as moe
    ws = torch.empty(1 << 16, dtype=torch.uint8, device="cuda")
    assert moe.moe_selftest_wait_timeout(ws, ws.numel(), 50_000) == moe.MOE_OK   # 50 ms limit
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_TIMEOUT
    assert int(ws[128:132].view(torch.int32).item()) == 2                        # both waits gave up
    # the context is intact: a layer call right after is correct and reports OK
    wl = synth.workload("tiny").generate()
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    layer = moe.MoELayer(torch.from_numpy(wl.Wg).cuda(), to_dev(wl.W1), to_dev(wl.W3), to_dev(wl.W2))
    y = layer.forward(to_dev(wl.x))
    assert layer.device_status(wl.T) == moe.MOE_OK
    ref = oracle.Oracle().layer(wl.x, wl.Wg, wl.W1, wl.W3, wl.W2, wl.k)["y"]
    got = synth.bf16_to_f32(y.cpu().view(torch.int16).numpy().view(np.uint16)).astype(np.float64)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 5e-3

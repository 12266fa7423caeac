"""Layer calls on several streams at once and inside CUDA graphs.

* Two layers, each with its own workspace, run interleaved on two streams
  with no host synchronisation between their calls; their kernels may
  overlap on the device.  No kernel of the library waits on another block
  except in ticket order, and all per-call state lives in the call's
  workspace, so each output equals the same call made alone, bit for bit.
* The capacity and next-best-fallback policies and the 4-bit layer queue
  more kernels and memsets than the dropless bf16 layer; captured in a CUDA
  graph, each replays to its eager output, bit for bit.
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


def _layer(wl, **kw):
    return moe.MoELayer(torch.from_numpy(wl.Wg).cuda(), H.to_dev_bf16(wl.W1), H.to_dev_bf16(wl.W3),
                        H.to_dev_bf16(wl.W2), k=wl.k, capacity_factor=wl.capacity_factor,
                        drop_policy=wl.drop_policy, **kw)


def test_two_streams_interleaved():
    """A 300-token batch (CTA-pair GEMMs) on one stream and a 64-token batch
    (streaming GEMMs) on another, three calls each, queued alternately."""
    wl = synth.Workload("streams", 300, 256, 512, seed=31).generate()
    la = _layer(wl)
    lb = moe.MoELayer(la.Wg, la.W1, la.W3, la.W2, k=wl.k)    # same weights, its own workspaces
    xa = [H.to_dev_bf16(synth.normal_bf16(40 + i, synth.TID_X, (300, wl.d))) for i in range(3)]
    xb = [H.to_dev_bf16(synth.normal_bf16(50 + i, synth.TID_X, (64, wl.d))) for i in range(3)]
    ref_a = [la.forward(x).clone() for x in xa]
    ref_b = [lb.forward(x).clone() for x in xb]
    torch.cuda.synchronize()
    ya = [torch.zeros_like(r) for r in ref_a]
    yb = [torch.zeros_like(r) for r in ref_b]
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    sa.wait_stream(torch.cuda.current_stream())
    sb.wait_stream(torch.cuda.current_stream())
    for i in range(3):
        with torch.cuda.stream(sa):
            la.forward(xa[i], ya[i])
        with torch.cuda.stream(sb):
            lb.forward(xb[i], yb[i])
    torch.cuda.synchronize()
    assert la.device_status(300) == moe.MOE_OK and lb.device_status(64) == moe.MOE_OK
    for i in range(3):
        assert torch.equal(ya[i].view(torch.int16), ref_a[i].view(torch.int16)), i
        assert torch.equal(yb[i].view(torch.int16), ref_b[i].view(torch.int16)), i


def _replay_matches_eager(layer, x, T):
    y_eager = layer.forward(x).clone()
    y = torch.empty_like(y_eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer.forward(x, y)          # first call on this stream outside capture
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    y.zero_()
    with torch.cuda.graph(g):
        layer.forward(x, y)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert layer.device_status(T) == moe.MOE_OK
    assert torch.equal(y.view(torch.int16), y_eager.view(torch.int16))
    del g


@pytest.mark.parametrize("policy", [0, 1, 2, 3], ids=["by_prob", "by_order", "by_prob_next", "by_order_next"])
def test_capacity_layer_replays_in_cuda_graph(policy):
    wl = synth.Workload("graphcap", 256, 128, 448, capacity_factor=1.0, drop_policy=policy, skew=True,
                        seed=13).generate()
    _replay_matches_eager(_layer(wl), H.to_dev_bf16(wl.x), wl.T)


@pytest.mark.parametrize("T", [16, 200])
def test_q4_layer_replays_in_cuda_graph(T):
    wl = synth.Workload("graphq4", T, 128, 448, seed=14).generate()
    q = [(torch.from_numpy(c).cuda(), H.to_dev_bf16(s)) for c, s in
         (oracle.Oracle().q4_quantize(W) for W in (wl.W1, wl.W3, wl.W2))]
    layer = moe.MoELayerQ4(torch.from_numpy(wl.Wg).cuda(), *q, k=wl.k)
    _replay_matches_eager(layer, H.to_dev_bf16(wl.x), T)

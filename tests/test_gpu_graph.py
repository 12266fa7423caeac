"""The whole layer captured in a CUDA graph: the library's calls queue
kernels, memsets and copies on the caller's stream (the chunked host-buffer
call also on its copy streams, forked from and joined to the caller's stream
by events), so a captured call replays to the same (bit-identical) output as
the eager call."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("variant", [1, 2, 3])
def test_layer_forward_replays_in_cuda_graph(variant):
    import sparse_mixture_experts_13_b200 as moe
    wl = synth.Workload("graph", 200, 128, 448, seed=12).generate()
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    layer = moe.MoELayer(torch.from_numpy(wl.Wg).cuda(), to_dev(wl.W1), to_dev(wl.W3), to_dev(wl.W2),
                         gemm_variant=variant)
    x = to_dev(wl.x)
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
    assert layer.device_status(wl.T) == moe.MOE_OK
    assert torch.equal(y.view(torch.int16), y_eager.view(torch.int16))


def test_chunked_host_call_replays_in_cuda_graph():
    """From 4096 dropless tokens moe_layer_forward_host runs the layer in
    token groups whose copies go through the library's copy streams, joined
    to the caller's stream by events.  Captured on the caller's stream, the
    call replays to the eager call's y bit for bit."""
    import sparse_mixture_experts_13_b200 as moe
    wl = synth.Workload("graph_host", 6000, 128, 256, seed=13).generate()
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    layer = moe.MoELayer(torch.from_numpy(wl.Wg).cuda(), to_dev(wl.W1), to_dev(wl.W3), to_dev(wl.W2))
    x_host = torch.from_numpy(np.ascontiguousarray(wl.x).view(np.int16)).view(torch.bfloat16).pin_memory()
    y_eager = torch.empty(wl.T, wl.d, dtype=torch.bfloat16).pin_memory()
    y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16).pin_memory()
    s = torch.cuda.Stream()
    layer.forward_host(x_host, y_eager, s)   # outside capture: workspace and copy streams exist
    torch.cuda.synchronize()
    y.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        layer.forward_host(x_host, y, s)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert layer.device_status(wl.T) == moe.MOE_OK
    assert torch.equal(y.view(torch.int16), y_eager.view(torch.int16))

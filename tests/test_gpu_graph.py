"""The whole layer captured in a CUDA graph: the library's calls queue only
kernels, memsets and copies on the caller's stream, so a captured call replays
to the same (bit-identical) output as the eager call."""
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

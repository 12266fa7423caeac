"""Host-side argument checks of the layer classes (no GPU needed).

The kernels read and write through raw pointers, so MoELayer and MoELayerQ4
refuse an activation that is not a contiguous bf16 [T, d] tensor on the
weights' device, and index outputs that are too small, before any work is
queued.  The layers are built here around CPU tensors (bypassing the CUDA
check of the constructor) so that the checks run on a host without a GPU; a
well-formed call then gets past them to the CUDA side.
"""
import pytest
import torch

from sparse_mixture_experts_13_b200.layer import MoELayer, MoELayerQ4, check_activation, check_index_out

T, D, F, E, K = 16, 128, 256, 8, 2


def _layer_cpu():
    L = MoELayer.__new__(MoELayer)
    L.Wg = torch.zeros(E, D, dtype=torch.float32)
    L.W1 = torch.zeros(E, F, D, dtype=torch.bfloat16)
    L.W3 = torch.zeros(E, F, D, dtype=torch.bfloat16)
    L.W2 = torch.zeros(E, D, F, dtype=torch.bfloat16)
    L.E, L.f, L.d, L.k = E, F, D, K
    L.capacity_factor, L.drop_policy, L.gemm_variant = 0.0, 0, 0
    L._ws = {}
    return L


def _layer_q4_cpu():
    L = MoELayerQ4.__new__(MoELayerQ4)
    L.Wg = torch.zeros(E, D, dtype=torch.float32)
    q = (torch.zeros(E, F, D // 2, dtype=torch.uint8), torch.zeros(E, D // 64, F, dtype=torch.bfloat16))
    L.q1 = L.q3 = q
    L.q2 = (torch.zeros(E, D, F // 2, dtype=torch.uint8), torch.zeros(E, F // 64, D, dtype=torch.bfloat16))
    L.E, L.f, L.d, L.k = E, F, D, K
    L.capacity_factor, L.drop_policy = 0.0, 0
    L._ws = {}
    return L


GOOD = lambda: torch.zeros(T, D, dtype=torch.bfloat16)
BAD_X = {
    "fp32": lambda: torch.zeros(T, D, dtype=torch.float32),
    "narrow": lambda: torch.zeros(T, D // 2, dtype=torch.bfloat16),
    "flat": lambda: torch.zeros(T * D, dtype=torch.bfloat16),
    "strided": lambda: torch.zeros(D, T, dtype=torch.bfloat16).t(),
    "3d": lambda: torch.zeros(T, D, 1, dtype=torch.bfloat16),
}


@pytest.mark.parametrize("cls", ["bf16", "q4"])
@pytest.mark.parametrize("bad", list(BAD_X))
def test_forward_refuses_malformed_x(cls, bad):
    L = _layer_cpu() if cls == "bf16" else _layer_q4_cpu()
    with pytest.raises(ValueError, match="x must be"):
        L.forward(BAD_X[bad]())


@pytest.mark.parametrize("cls", ["bf16", "q4"])
def test_forward_refuses_malformed_outputs(cls):
    L = _layer_cpu() if cls == "bf16" else _layer_q4_cpu()
    with pytest.raises(ValueError, match="y must be"):
        L.forward(GOOD(), torch.zeros(T - 1, D, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="topk_idx"):
        L.forward(GOOD(), topk_idx=torch.zeros(T * K - 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="topk_idx"):
        L.forward(GOOD(), topk_idx=torch.zeros(T * K, dtype=torch.int64))
    with pytest.raises(ValueError, match="counts"):
        L.forward(GOOD(), counts=torch.zeros(E - 1, dtype=torch.int32))


@pytest.mark.parametrize("cls", ["bf16", "q4"])
def test_wellformed_call_passes_the_checks(cls):
    """A well-formed call gets past the checks to the CUDA side, which is
    absent here (on a GPU host this is the normal path, covered by the GPU
    tests): the error is CUDA's or the library's, not a ValueError."""
    if torch.cuda.is_available():
        pytest.skip("host without a GPU only")
    L = _layer_cpu() if cls == "bf16" else _layer_q4_cpu()
    with pytest.raises(RuntimeError) as exc:
        L.forward(GOOD(), GOOD(), topk_idx=torch.zeros(T * K, dtype=torch.int32),
                  counts=torch.zeros(E, dtype=torch.int32))
    assert not isinstance(exc.value, ValueError)


def test_forward_host_refuses_device_or_malformed_buffers():
    L = _layer_cpu()
    with pytest.raises(ValueError, match="y_host must be"):
        L.forward_host(GOOD(), torch.zeros(T, D + 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="x_host must be"):
        L.forward_host(torch.zeros(T, D, dtype=torch.float16), GOOD())


def test_check_helpers_name_the_problem():
    with pytest.raises(ValueError, match=r"\[4, 64\].*got \(4, 32\)"):
        check_activation(torch.zeros(4, 32, dtype=torch.bfloat16), 4, 64, torch.device("cpu"), "x")
    with pytest.raises(ValueError, match="got list"):
        check_activation([1, 2], 4, 64, torch.device("cpu"), "x")
    check_activation(torch.zeros(4, 64, dtype=torch.bfloat16), 4, 64, torch.device("cpu"), "x")
    check_index_out(None, 8, torch.device("cpu"), "counts")
    check_index_out(torch.zeros(9, dtype=torch.int32), 8, torch.device("cpu"), "counts")

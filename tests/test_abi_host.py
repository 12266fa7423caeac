"""Host-side checks of the C ABI that need no GPU: the library builds and
loads, exports every entry point include/moe.h declares, and rejects bad
arguments with the documented status before touching a device."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def moe():
    from sparse_mixture_experts_13_b200 import build as b
    b.build()
    import sparse_mixture_experts_13_b200 as m
    return m


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)))


def test_exports_match_header(moe):
    names = declared_symbols()
    assert len(names) >= 9, names
    lib = ctypes.CDLL(moe._lib.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(moe.EXPORTED) == names


def test_binding_constants_match_header(moe):
    """Every enum value include/moe.h declares has the same value in the binding."""
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    vals = re.findall(r"\b(MOE_[A-Z0-9_]+)\s*=\s*(\d+)", src)
    assert len(vals) >= 14, vals
    for name, v in vals:
        assert getattr(moe, name) == int(v), name


def test_shape_struct_layout(moe):
    assert ctypes.sizeof(moe.moe_shape) == 40
    assert moe.moe_shape.capacity_factor.offset == 24


def test_status_strings(moe):
    for code in range(6):
        assert moe.status_string(code)
    assert moe.status_string(99) == "unknown status"


@pytest.mark.parametrize("kw", [dict(E=0), dict(E=33), dict(k=0), dict(k=9, E=16), dict(k=3, E=2),
                                dict(d_model=100), dict(d_model=0), dict(d_ff=448 + 32), dict(T=-1),
                                dict(capacity_factor=float("nan")), dict(capacity_factor=float("inf")),
                                dict(drop_policy=4), dict(drop_policy=-1), dict(gemm_variant=4), dict(T=1 << 29, k=2)])
def test_invalid_shapes(moe, kw):
    base = dict(T=64, d_model=128, d_ff=448, E=8, k=2)
    base.update(kw)
    sh = moe.make_shape(**base)
    assert moe.moe_workspace_size(sh) == 0
    assert moe.moe_layer_forward(sh, 16, 16, 16, 16, 16, 16, None, None, 256, 1 << 40, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_router_topk(sh, 16, 16, None, 16, 16, 16, 16, 0) == moe.MOE_ERR_INVALID_ARG


def test_workspace_size(moe):
    sizes = [moe.moe_workspace_size(moe.make_shape(T, 4096, 14336)) for T in (1, 16, 129, 4096)]
    assert all(s > 0 for s in sizes) and sizes == sorted(sizes)
    prefill = moe.moe_workspace_size(moe.make_shape(4096, 4096, 14336))
    # at least x_perm + h + y_perm for T*k rows
    assert prefill >= 8192 * (4096 * 2 * 2 + 14336 * 2)
    assert moe.moe_workspace_size(moe.make_shape(0, 128, 448)) > 0


def test_bad_pointers_rejected_before_device(moe):
    sh = moe.make_shape(64, 128, 448)
    ws_n = moe.moe_workspace_size(sh)
    ok = 1 << 20  # an aligned fake address: never dereferenced on these paths
    E = moe.MOE_ERR_INVALID_ARG
    assert moe.moe_router_topk(sh, None, ok, None, ok, ok, ok, ok, 0) == E
    assert moe.moe_router_topk(sh, ok + 2, ok, None, ok, ok, ok, ok, 0) == E       # x misaligned
    assert moe.moe_router_topk(sh, ok, ok, ok + 1, ok, ok, ok, ok, 0) == E          # logits misaligned
    assert moe.moe_combine(sh, ok, ok, ok, ok + 8, 0) == E                          # y misaligned
    assert moe.moe_grouped_swiglu(sh, ok, ok, ok, ok, None, ok, ok, ok, ws_n, 0) == E
    W = moe.MOE_ERR_WORKSPACE
    assert moe.moe_permute(sh, ok, ok, ok, ok, ok, ok, ok, ok, None, ws_n, 0) == W
    assert moe.moe_permute(sh, ok, ok, ok, ok, ok, ok, ok, ok, ok + 128, ws_n, 0) == W
    assert moe.moe_permute(sh, ok, ok, ok, ok, ok, ok, ok, ok, ok, ws_n - 1, 0) == W
    assert moe.moe_layer_forward(sh, ok, ok, ok, ok, ok, ok, None, None, ok, ws_n - 256, 0) == W
    assert moe.moe_layer_forward_host(sh, None, ok, ok, ok, ok, ok, ok, ws_n, 0) == E
    assert moe.moe_read_device_status(None, 0) == W
    # T == 0 is a no-op whatever the pointers
    sh0 = moe.make_shape(0, 128, 448)
    assert moe.moe_layer_forward(sh0, None, None, None, None, None, None, None, None, None, 0, 0) == moe.MOE_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_reports_cuda_error(moe):
    sh = moe.make_shape(64, 128, 448)
    ok = 1 << 20
    st = moe.moe_router_topk(sh, ok, ok, None, ok, ok, ok, ok, 0)
    assert st in (moe.MOE_ERR_CUDA, moe.MOE_ERR_UNSUPPORTED)


def test_selftest_arguments(moe):
    ok = 1 << 20
    assert moe.moe_selftest_wait_timeout(None, 1 << 16, 1000, 0) == moe.MOE_ERR_WORKSPACE
    assert moe.moe_selftest_wait_timeout(ok + 16, 1 << 16, 1000, 0) == moe.MOE_ERR_WORKSPACE
    assert moe.moe_selftest_wait_timeout(ok, 128, 1000, 0) == moe.MOE_ERR_WORKSPACE
    assert moe.moe_selftest_wait_timeout(ok, 1 << 16, 0, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_selftest_wait_timeout(ok, 1 << 16, 20_000_000, 0) == moe.MOE_ERR_INVALID_ARG


def test_q4_arguments_rejected_before_device(moe):
    sh = moe.make_shape(64, 128, 448)
    assert moe.moe_workspace_size_q4(moe.make_shape(64, 100, 448)) == 0
    n = moe.moe_workspace_size_q4(sh)
    assert n > 0
    ok = 1 << 20
    q = (ok, ok)
    E, W = moe.MOE_ERR_INVALID_ARG, moe.MOE_ERR_WORKSPACE
    assert moe.moe_layer_forward_q4(sh, ok, ok, (None, ok), q, q, ok, None, None, ok, n, 0) == E
    assert moe.moe_layer_forward_q4(sh, ok, ok, q, (ok, ok + 2), q, ok, None, None, ok, n, 0) == E
    assert moe.moe_layer_forward_q4(sh, ok, ok, q, q, q, ok, None, None, ok, n - 1, 0) == W
    assert moe.moe_grouped_swiglu_q4(sh, ok, ok, q, q, (ok + 8, ok), ok, ok, ok, n, 0) == E
    assert moe.moe_layer_forward_q4_profiled(sh, ok, ok, q, q, q, ok, [ok] * 6, None, n, 0) == W
    assert moe.moe_layer_forward_q4_host(sh, None, ok, q, q, q, ok, ok, n, 0) == E
    assert moe.moe_layer_forward_q4_host(sh, ok, ok, q, q, q, None, ok, n, 0) == E
    assert moe.moe_layer_forward_q4_host(sh, ok, ok, (ok + 4, ok), q, q, ok, ok, n, 0) == E
    assert moe.moe_layer_forward_q4_host(sh, ok, ok, q, q, q, ok, ok, n - 1, 0) == W
    assert moe.moe_layer_forward_q4_host(moe.make_shape(0, 128, 448), None, None, (None, None), (None, None),
                                         (None, None), None, None, 0, 0) == moe.MOE_OK
    for bad in ((0, 64, 128), (2, 60, 128), (2, 64, 96), (33, 64, 128), (2, 64, 65600)):
        assert moe.moe_quantize_q4(ok, *bad, ok, ok, 0) == E
    assert moe.moe_quantize_q4(ok, 2, 64, 128, ok + 4, ok, 0) == E
    # T == 0 is a no-op
    assert moe.moe_layer_forward_q4(moe.make_shape(0, 128, 448), None, None, (None, None), (None, None),
                                    (None, None), None, None, None, None, 0, 0) == moe.MOE_OK


def test_q4_workspace_holds_partials(moe):
    for T in (1, 16, 129, 4096):
        sh = moe.make_shape(T, 4096, 14336)
        assert moe.moe_workspace_size_q4(sh) >= T * 2 * 4096 * 4  # at least one fp32 partial buffer


def test_router_stats_arguments(moe):
    sh = moe.make_shape(64, 128, 448)
    ok = 1 << 20
    E = moe.MOE_ERR_INVALID_ARG
    assert moe.moe_router_stats(sh, ok, None, None, 0, 0) == E          # slot_counts missing
    assert moe.moe_router_stats(sh, None, ok, None, 0, 0) == E          # topk_idx missing
    assert moe.moe_router_stats(sh, ok, ok + 2, None, 0, 0) == E        # misaligned
    assert moe.moe_router_stats(sh, ok, ok, ok, 2, 0) == E              # accumulate flag
    assert moe.moe_router_stats(moe.make_shape(64, 128, 448, E=8, k=1), ok, ok, ok, 0, 0) == E  # pairs need k >= 2
    assert moe.moe_router_stats(moe.make_shape(64, 100, 448), ok, ok, None, 0, 0) == E


def test_fallback_policies_accepted(moe):
    """Policies 2 and 3 (next-best-expert fallback) are valid shapes; the
    whole layer takes them, and their workspace holds the fallback's arrays."""
    plain = moe.moe_workspace_size(moe.make_shape(256, 128, 448, capacity_factor=1.0, drop_policy=0))
    for pol in (2, 3):
        sh = moe.make_shape(256, 128, 448, capacity_factor=1.0, drop_policy=pol)
        assert moe.moe_workspace_size(sh) > plain
        assert moe.moe_workspace_size_q4(sh) > 0
    # dropless ignores the policy
    assert moe.moe_workspace_size(moe.make_shape(256, 128, 448, drop_policy=2)) == \
        moe.moe_workspace_size(moe.make_shape(256, 128, 448))


def test_fallback_rejected_by_stage_permute(moe):
    """The next-best fallback needs the router's ranks past the top k, which
    only the whole-layer entry points compute: the stage grouping entry points
    refuse those policies before touching a device."""
    ok = 1 << 20
    for pol in (2, 3):
        sh = moe.make_shape(64, 128, 448, capacity_factor=1.0, drop_policy=pol)
        n = moe.moe_workspace_size(sh)
        assert moe.moe_permute(sh, ok, ok, ok, ok, ok, ok, ok, ok, ok, n, 0) == moe.MOE_ERR_UNSUPPORTED
        assert moe.moe_permute_noalloc(sh, ok, ok, ok, ok, ok, ok, ok, ok, 0) == moe.MOE_ERR_UNSUPPORTED
    # dropless with the same policy value is an ordinary grouping (no fallback to take)
    sh0 = moe.make_shape(64, 128, 448, drop_policy=2)
    assert moe.moe_permute(sh0, ok, ok, ok, ok, ok, ok, ok, ok, None, 0, 0) == moe.MOE_ERR_WORKSPACE

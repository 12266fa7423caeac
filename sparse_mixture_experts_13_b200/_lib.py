"""ctypes binding of ``libmoe.so`` (the C ABI in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Tensors are passed by ``data_ptr()``; ``None`` becomes NULL;
plain integers are taken as addresses.  Each wrapper returns the library's
``moe_status`` code (0 = MOE_OK); ``check()`` turns a non-zero code into
``MoeError``.  There is no fallback: if the library is missing the first call
raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_LIB=debug selects the debug build (device-side bounds checks, workspace
# guards, stage-failure hook); the default is the release library.
LIB_PATH = os.path.join(_PKG, "libmoe_debug.so" if os.environ.get("MOE_LIB") == "debug" else "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, \
    MOE_ERR_BOUNDS = range(7)
MOE_DROP_BY_PROB, MOE_DROP_BY_ORDER, MOE_DROP_BY_PROB_NEXT_BEST, MOE_DROP_BY_ORDER_NEXT_BEST = 0, 1, 2, 3
MOE_VARIANT_AUTO, MOE_VARIANT_TILED, MOE_VARIANT_STREAM, MOE_VARIANT_TILED_SINGLE = 0, 1, 2, 3

EXPORTED = ("moe_workspace_size", "moe_router_topk", "moe_permute", "moe_grouped_swiglu", "moe_combine",
            "moe_layer_forward", "moe_layer_forward_host", "moe_layer_forward_profiled", "moe_permute_noalloc",
            "moe_permute_noalloc_status",
            "moe_selftest_wait_timeout", "moe_read_device_status", "moe_router_stats", "moe_ep_plan", "moe_ep_dispatch",
            "moe_ep_combine", "moe_ep_dispatch_cap", "moe_ep_select", "moe_ep_combine_cap", "moe_quantize_q4", "moe_workspace_size_q4",
            "moe_grouped_swiglu_q4", "moe_layer_forward_q4", "moe_layer_forward_q4_profiled", "moe_layer_forward_q4_host",
            "moe_debug_build", "moe_debug_workspace_arm", "moe_debug_workspace_check", "moe_status_string")
_SIZE_RETURNING = ("moe_workspace_size", "moe_workspace_size_q4")


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class moe_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("capacity_factor", ctypes.c_float),
                ("drop_policy", ctypes.c_int32), ("gemm_variant", ctypes.c_int32)]


def make_shape(T, d_model, d_ff, E=8, k=2, capacity_factor=0.0, drop_policy=0, gemm_variant=0) -> moe_shape:
    return moe_shape(int(T), int(d_model), int(d_ff), int(E), int(k), float(capacity_factor),
                     int(drop_policy), int(gemm_variant))


_lib = None


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmoe.so is not built ({LIB_PATH}); run the package build first")
        L = ctypes.CDLL(LIB_PATH)
        P, S, st = ctypes.c_void_p, ctypes.POINTER(moe_shape), ctypes.c_int
        sz = ctypes.c_size_t
        L.moe_workspace_size.argtypes = [S]
        L.moe_workspace_size.restype = sz
        L.moe_router_topk.argtypes = [S, P, P, P, P, P, P, P, P]
        L.moe_permute.argtypes = [S, P, P, P, P, P, P, P, P, P, sz, P]
        L.moe_permute_noalloc.argtypes = [S, P, P, P, P, P, P, P, P, P]
        L.moe_permute_noalloc_status.argtypes = [P]
        L.moe_grouped_swiglu.argtypes = [S, P, P, P, P, P, P, P, P, sz, P]
        L.moe_combine.argtypes = [S, P, P, P, P, P]
        L.moe_layer_forward.argtypes = [S, P, P, P, P, P, P, P, P, P, sz, P]
        L.moe_layer_forward_host.argtypes = [S, P, P, P, P, P, P, P, sz, P]
        L.moe_layer_forward_profiled.argtypes = [S, P, P, P, P, P, P, P, P, sz, P]
        L.moe_read_device_status.argtypes = [P, P]
        L.moe_selftest_wait_timeout.argtypes = [P, sz, ctypes.c_uint32, P]
        L.moe_router_stats.argtypes = [S, P, P, P, ctypes.c_int32, P]
        i32 = ctypes.c_int32
        L.moe_ep_plan.argtypes = [P, i32, i32, i32, P, P, P]
        L.moe_ep_dispatch.argtypes = [S, i32, P, P, P, P, P, P, P, sz, P]
        L.moe_ep_combine.argtypes = [S, i32, P, P, P, P, P, P]
        L.moe_ep_dispatch_cap.argtypes = [S, i32, i32, P, P, P, P, P, P, P, P, P, P, sz, P]
        L.moe_ep_select.argtypes = [S, i32, P, P, P, P, P, P, P, P]
        L.moe_ep_combine_cap.argtypes = [S, i32, P, P, P, P, P, P, P]
        L.moe_quantize_q4.argtypes = [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, P, P]
        L.moe_workspace_size_q4.argtypes = [S]
        L.moe_grouped_swiglu_q4.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, sz, P]
        L.moe_layer_forward_q4.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, sz, P]
        L.moe_layer_forward_q4_profiled.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, sz, P]
        L.moe_layer_forward_q4_host.argtypes = [S, P, P, P, P, P, P, P, P, P, P, sz, P]
        L.moe_debug_build.argtypes = []
        L.moe_debug_workspace_arm.argtypes = [S, P, sz, ctypes.c_int32, P]
        L.moe_debug_workspace_check.argtypes = [S, P, sz, ctypes.c_int32, P]
        L.moe_status_string.argtypes = [st]
        L.moe_status_string.restype = ctypes.c_char_p
        for name in EXPORTED:
            if name in _SIZE_RETURNING:
                getattr(L, name).restype = sz
            elif name != "moe_status_string":
                getattr(L, name).restype = st
        _lib = L
    return _lib


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def check(status: int, what: str = "moe") -> None:
    if status != MOE_OK:
        raise MoeError(status, what)


def moe_workspace_size(shape: moe_shape) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(shape)))


def moe_router_topk(shape, x, Wg, logits, topk_idx, topk_w, topk_p, counts, stream=None) -> int:
    return lib().moe_router_topk(ctypes.byref(shape), _p(x), _p(Wg), _p(logits), _p(topk_idx), _p(topk_w),
                                 _p(topk_p), _p(counts), _stream(stream))


def moe_permute(shape, x, topk_idx, topk_p, counts, offsets, slot_pos, perm_slot, x_perm, ws, ws_bytes,
                stream=None) -> int:
    return lib().moe_permute(ctypes.byref(shape), _p(x), _p(topk_idx), _p(topk_p), _p(counts), _p(offsets),
                             _p(slot_pos), _p(perm_slot), _p(x_perm), _p(ws), int(ws_bytes), _stream(stream))


def moe_permute_noalloc(shape, x, topk_idx, topk_p, counts, offsets, slot_pos, perm_slot, x_perm,
                        stream=None) -> int:
    """moe_permute with its scratch in a fixed device array (no workspace)."""
    return lib().moe_permute_noalloc(ctypes.byref(shape), _p(x), _p(topk_idx), _p(topk_p), _p(counts), _p(offsets),
                                     _p(slot_pos), _p(perm_slot), _p(x_perm), _stream(stream))


def moe_permute_noalloc_status(stream=None) -> int:
    """Status of the last moe_permute_noalloc call on the current device."""
    return lib().moe_permute_noalloc_status(_stream(stream))


def moe_grouped_swiglu(shape, x_perm, offsets, W1, W3, W2, h, y_perm, ws, ws_bytes, stream=None) -> int:
    return lib().moe_grouped_swiglu(ctypes.byref(shape), _p(x_perm), _p(offsets), _p(W1), _p(W3), _p(W2), _p(h),
                                    _p(y_perm), _p(ws), int(ws_bytes), _stream(stream))


def moe_combine(shape, y_perm, slot_pos, topk_w, y, stream=None) -> int:
    return lib().moe_combine(ctypes.byref(shape), _p(y_perm), _p(slot_pos), _p(topk_w), _p(y), _stream(stream))


def moe_layer_forward(shape, x, Wg, W1, W3, W2, y, topk_idx_out, counts_out, ws, ws_bytes, stream=None) -> int:
    return lib().moe_layer_forward(ctypes.byref(shape), _p(x), _p(Wg), _p(W1), _p(W3), _p(W2), _p(y),
                                   _p(topk_idx_out), _p(counts_out), _p(ws), int(ws_bytes), _stream(stream))


def moe_layer_forward_host(shape, x_host, Wg, W1, W3, W2, y_host, ws, ws_bytes, stream=None) -> int:
    return lib().moe_layer_forward_host(ctypes.byref(shape), _p(x_host), _p(Wg), _p(W1), _p(W3), _p(W2),
                                        _p(y_host), _p(ws), int(ws_bytes), _stream(stream))


def moe_layer_forward_profiled(shape, x, Wg, W1, W3, W2, y, events, ws, ws_bytes, stream=None) -> int:
    """events: six torch.cuda.Event(enable_timing=True) objects (or raw handles)."""
    arr = _event_handles(events)
    return lib().moe_layer_forward_profiled(ctypes.byref(shape), _p(x), _p(Wg), _p(W1), _p(W3), _p(W2), _p(y), arr,
                                            _p(ws), int(ws_bytes), _stream(stream))


def _event_handles(events):
    handles = []
    for ev in events:
        if isinstance(ev, int):
            handles.append(ev)
        else:
            if ev.cuda_event == 0:
                ev.record()  # creates the underlying event
            handles.append(ev.cuda_event)
    return (ctypes.c_void_p * 6)(*handles)


def moe_router_stats(shape, topk_idx, slot_counts, pair_counts=None, accumulate=0, stream=None) -> int:
    """Per-slot expert histograms [k, E] and first-two-choice pair counts [E, E]."""
    return lib().moe_router_stats(ctypes.byref(shape), _p(topk_idx), _p(slot_counts), _p(pair_counts),
                                  int(accumulate), _stream(stream))


# ------------------------------------------------------ expert parallelism
# peer_x / peer_y: int64 CUDA tensors holding one device pointer per rank.

def moe_ep_plan(counts_all, E, rank, world, recv_off, owner_off, stream=None) -> int:
    return lib().moe_ep_plan(_p(counts_all), int(E), int(rank), int(world), _p(recv_off), _p(owner_off),
                             _stream(stream))


def moe_ep_dispatch(shape, world, x, topk_idx, counts, recv_off, peer_x, ret_row, ws, ws_bytes, stream=None) -> int:
    return lib().moe_ep_dispatch(ctypes.byref(shape), int(world), _p(x), _p(topk_idx), _p(counts), _p(recv_off),
                                 _p(peer_x), _p(ret_row), _p(ws), int(ws_bytes), _stream(stream))


def moe_ep_combine(shape, world, topk_idx, topk_w, ret_row, peer_y, y, stream=None) -> int:
    return lib().moe_ep_combine(ctypes.byref(shape), int(world), _p(topk_idx), _p(topk_w), _p(ret_row), _p(peer_y),
                                _p(y), _stream(stream))


def moe_ep_dispatch_cap(shape, world, rank, counts_all, x, topk_idx, topk_p, counts, recv_off, peer_x, peer_keys,
                        ret_row, ws, ws_bytes, stream=None) -> int:
    return lib().moe_ep_dispatch_cap(ctypes.byref(shape), int(world), int(rank), _p(counts_all), _p(x), _p(topk_idx),
                                     _p(topk_p), _p(counts), _p(recv_off), _p(peer_x), _p(peer_keys), _p(ret_row),
                                     _p(ws), int(ws_bytes), _stream(stream))


def moe_ep_select(shape, world, counts_all, owner_off, keys, x_recv, x_kept, kept_off, row_map, stream=None) -> int:
    return lib().moe_ep_select(ctypes.byref(shape), int(world), _p(counts_all), _p(owner_off), _p(keys), _p(x_recv),
                               _p(x_kept), _p(kept_off), _p(row_map), _stream(stream))


def moe_ep_combine_cap(shape, world, topk_idx, topk_w, ret_row, peer_map, peer_y, y, stream=None) -> int:
    return lib().moe_ep_combine_cap(ctypes.byref(shape), int(world), _p(topk_idx), _p(topk_w), _p(ret_row),
                                    _p(peer_map), _p(peer_y), _p(y), _stream(stream))


# ------------------------------------------------------------ 4-bit experts
# A 4-bit matrix is passed as a (codes, scales) pair: codes [E, R, K/2] uint8,
# scales [E, K/64, R] bf16 bits.

def moe_quantize_q4(W, E, R, K, codes, scales, stream=None) -> int:
    return lib().moe_quantize_q4(_p(W), int(E), int(R), int(K), _p(codes), _p(scales), _stream(stream))


def moe_workspace_size_q4(shape: moe_shape) -> int:
    return int(lib().moe_workspace_size_q4(ctypes.byref(shape)))


def moe_grouped_swiglu_q4(shape, x_perm, offsets, q1, q3, q2, h, y_perm, ws, ws_bytes, stream=None) -> int:
    return lib().moe_grouped_swiglu_q4(ctypes.byref(shape), _p(x_perm), _p(offsets), _p(q1[0]), _p(q1[1]),
                                       _p(q3[0]), _p(q3[1]), _p(q2[0]), _p(q2[1]), _p(h), _p(y_perm), _p(ws),
                                       int(ws_bytes), _stream(stream))


def moe_layer_forward_q4(shape, x, Wg, q1, q3, q2, y, topk_idx_out, counts_out, ws, ws_bytes, stream=None) -> int:
    return lib().moe_layer_forward_q4(ctypes.byref(shape), _p(x), _p(Wg), _p(q1[0]), _p(q1[1]), _p(q3[0]),
                                      _p(q3[1]), _p(q2[0]), _p(q2[1]), _p(y), _p(topk_idx_out), _p(counts_out),
                                      _p(ws), int(ws_bytes), _stream(stream))


def moe_layer_forward_q4_host(shape, x_host, Wg, q1, q3, q2, y_host, ws, ws_bytes, stream=None) -> int:
    return lib().moe_layer_forward_q4_host(ctypes.byref(shape), _p(x_host), _p(Wg), _p(q1[0]), _p(q1[1]),
                                           _p(q3[0]), _p(q3[1]), _p(q2[0]), _p(q2[1]), _p(y_host), _p(ws),
                                           int(ws_bytes), _stream(stream))


def moe_layer_forward_q4_profiled(shape, x, Wg, q1, q3, q2, y, events, ws, ws_bytes, stream=None) -> int:
    return lib().moe_layer_forward_q4_profiled(ctypes.byref(shape), _p(x), _p(Wg), _p(q1[0]), _p(q1[1]),
                                               _p(q3[0]), _p(q3[1]), _p(q2[0]), _p(q2[1]), _p(y),
                                               _event_handles(events), _p(ws), int(ws_bytes), _stream(stream))


def moe_selftest_wait_timeout(ws, ws_bytes, limit_us, stream=None) -> int:
    return lib().moe_selftest_wait_timeout(_p(ws), int(ws_bytes), int(limit_us), _stream(stream))


def moe_read_device_status(ws, stream=None) -> int:
    return lib().moe_read_device_status(_p(ws), _stream(stream))


# ------------------------------------------------------------ debug build

def moe_debug_build() -> int:
    return int(lib().moe_debug_build())


def moe_debug_workspace_arm(shape, ws, ws_bytes, q4=False, stream=None) -> int:
    return lib().moe_debug_workspace_arm(ctypes.byref(shape), _p(ws), int(ws_bytes), int(bool(q4)), _stream(stream))


def moe_debug_workspace_check(shape, ws, ws_bytes, q4=False, stream=None) -> int:
    return lib().moe_debug_workspace_check(ctypes.byref(shape), _p(ws), int(ws_bytes), int(bool(q4)),
                                           _stream(stream))

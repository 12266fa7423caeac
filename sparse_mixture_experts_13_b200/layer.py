"""Convenience holder of one MoE layer's device weights and workspace.

PyTorch provides the device memory and the stream; the computation is the
library's ``moe_layer_forward`` (or ``moe_layer_forward_host``).
"""
from __future__ import annotations

import torch

from . import _lib


def check_activation(t: torch.Tensor, T: int, d: int, device, name: str) -> None:
    """Raise ValueError unless `t` is a contiguous bf16 [T, d] tensor on
    `device`.  The kernels read and write exactly T * d elements through the
    raw pointer, so a smaller or differently placed tensor must be refused
    before anything is queued."""
    if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.dim() != 2 or \
            tuple(t.shape) != (T, d) or not t.is_contiguous() or t.device != device:
        got = (f"{tuple(t.shape)} {t.dtype} on {t.device}, contiguous={t.is_contiguous()}"
               if isinstance(t, torch.Tensor) else type(t).__name__)
        raise ValueError(f"{name} must be a contiguous bf16 [{T}, {d}] tensor on {device}; got {got}")


def check_index_out(t, n: int, device, name: str) -> None:
    """Raise ValueError unless `t` (optional) is a contiguous int32 tensor of
    at least n elements on `device`."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or t.dtype != torch.int32 or not t.is_contiguous() or \
            t.numel() < n or t.device != device:
        raise ValueError(f"{name} must be a contiguous int32 tensor of at least {n} elements on {device}")


class MoELayer:
    """Weights on one CUDA device: Wg [E, d] fp32, W1/W3 [E, f, d] and
    W2 [E, d, f] bf16 (row-major, contiguous)."""

    def __init__(self, Wg: torch.Tensor, W1: torch.Tensor, W3: torch.Tensor, W2: torch.Tensor, k: int = 2,
                 capacity_factor: float = 0.0, drop_policy: int = _lib.MOE_DROP_BY_PROB,
                 gemm_variant: int = _lib.MOE_VARIANT_AUTO):
        for t, dt in ((Wg, torch.float32), (W1, torch.bfloat16), (W3, torch.bfloat16), (W2, torch.bfloat16)):
            if t.dtype != dt or not t.is_cuda or not t.is_contiguous():
                raise ValueError("weights must be contiguous CUDA tensors (Wg fp32, W1/W3/W2 bf16)")
        self.Wg, self.W1, self.W3, self.W2 = Wg, W1, W3, W2
        self.E, self.f, self.d = W1.shape
        self.k = k
        self.capacity_factor = capacity_factor
        self.drop_policy = drop_policy
        self.gemm_variant = gemm_variant
        self._ws = {}

    def shape(self, T: int) -> _lib.moe_shape:
        return _lib.make_shape(T, self.d, self.f, self.E, self.k, self.capacity_factor, self.drop_policy,
                               self.gemm_variant)

    def workspace(self, T: int) -> torch.Tensor:
        ws = self._ws.get(T)
        if ws is None:
            n = _lib.moe_workspace_size(self.shape(T))
            if n == 0:
                raise ValueError("invalid layer shape")
            ws = torch.empty(n, dtype=torch.uint8, device=self.W1.device)
            self._ws[T] = ws
        return ws

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, topk_idx: torch.Tensor | None = None,
                counts: torch.Tensor | None = None) -> torch.Tensor:
        T = x.shape[0]
        dev = self.W1.device
        check_activation(x, T, self.d, dev, "x")
        if y is None:
            y = torch.empty((T, self.d), dtype=torch.bfloat16, device=x.device)
        check_activation(y, T, self.d, dev, "y")
        check_index_out(topk_idx, T * self.k, dev, "topk_idx")
        check_index_out(counts, self.E, dev, "counts")
        ws = self.workspace(T)
        st = _lib.moe_layer_forward(self.shape(T), x, self.Wg, self.W1, self.W3, self.W2, y, topk_idx, counts,
                                    ws, ws.numel())
        _lib.check(st, "moe_layer_forward")
        return y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, stream=None) -> None:
        """x_host, y_host: page-locked CPU bf16 [T, d]; queued on the stream."""
        T = x_host.shape[0]
        cpu = torch.device("cpu")
        check_activation(x_host, T, self.d, cpu, "x_host")
        check_activation(y_host, T, self.d, cpu, "y_host")
        ws = self.workspace(T)
        st = _lib.moe_layer_forward_host(self.shape(T), x_host, self.Wg, self.W1, self.W3, self.W2, y_host, ws,
                                         ws.numel(), stream)
        _lib.check(st, "moe_layer_forward_host")

    def device_status(self, T: int) -> int:
        return _lib.moe_read_device_status(self.workspace(T))


class MoELayerQ4:
    """One MoE layer with 4-bit expert weights on one CUDA device: Wg [E, d]
    fp32 and, per expert matrix, a (codes, scales) pair -- codes [E, R, K/2]
    uint8, scales [E, K/64, R] bf16 (W1, W3: R = d_ff, K = d_model; W2: R =
    d_model, K = d_ff).  The computation is ``moe_layer_forward_q4``."""

    def __init__(self, Wg: torch.Tensor, q1, q3, q2, k: int = 2, capacity_factor: float = 0.0,
                 drop_policy: int = _lib.MOE_DROP_BY_PROB):
        for c, s in (q1, q3, q2):
            if c.dtype != torch.uint8 or s.dtype != torch.bfloat16 or not (c.is_cuda and s.is_cuda) or \
                    not (c.is_contiguous() and s.is_contiguous()):
                raise ValueError("4-bit weights must be contiguous CUDA (uint8 codes, bf16 scales) pairs")
        if Wg.dtype != torch.float32 or not Wg.is_cuda or not Wg.is_contiguous():
            raise ValueError("Wg must be a contiguous CUDA fp32 tensor")
        self.Wg, self.q1, self.q3, self.q2 = Wg, q1, q3, q2
        self.E, self.f, half_d = q1[0].shape
        self.d = 2 * half_d
        self.k = k
        self.capacity_factor = capacity_factor
        self.drop_policy = drop_policy
        self._ws = {}

    @staticmethod
    def quantize_matrix(W: torch.Tensor, stream=None):
        """bf16 [E, R, K] on the device -> (codes, scales) with moe_quantize_q4."""
        E, R, K = W.shape
        codes = torch.empty(E, R, K // 2, dtype=torch.uint8, device=W.device)
        scales = torch.empty(E, K // 64, R, dtype=torch.bfloat16, device=W.device)
        _lib.check(_lib.moe_quantize_q4(W, E, R, K, codes, scales, stream), "moe_quantize_q4")
        return codes, scales

    @classmethod
    def from_bf16(cls, Wg, W1, W3, W2, **kw) -> "MoELayerQ4":
        q = [cls.quantize_matrix(W) for W in (W1, W3, W2)]
        return cls(Wg, *q, **kw)

    def shape(self, T: int) -> _lib.moe_shape:
        return _lib.make_shape(T, self.d, self.f, self.E, self.k, self.capacity_factor, self.drop_policy)

    def workspace(self, T: int) -> torch.Tensor:
        ws = self._ws.get(T)
        if ws is None:
            n = _lib.moe_workspace_size_q4(self.shape(T))
            if n == 0:
                raise ValueError("invalid layer shape")
            ws = torch.empty(n, dtype=torch.uint8, device=self.Wg.device)
            self._ws[T] = ws
        return ws

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, topk_idx: torch.Tensor | None = None,
                counts: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        dev = self.Wg.device
        check_activation(x, T, self.d, dev, "x")
        if y is None:
            y = torch.empty((T, self.d), dtype=torch.bfloat16, device=x.device)
        check_activation(y, T, self.d, dev, "y")
        check_index_out(topk_idx, T * self.k, dev, "topk_idx")
        check_index_out(counts, self.E, dev, "counts")
        ws = self.workspace(T)
        st = _lib.moe_layer_forward_q4(self.shape(T), x, self.Wg, self.q1, self.q3, self.q2, y, topk_idx, counts,
                                       ws, ws.numel(), stream)
        _lib.check(st, "moe_layer_forward_q4")
        return y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, stream=None) -> None:
        """x_host, y_host: page-locked CPU bf16 [T, d]; queued on the stream."""
        T = x_host.shape[0]
        cpu = torch.device("cpu")
        check_activation(x_host, T, self.d, cpu, "x_host")
        check_activation(y_host, T, self.d, cpu, "y_host")
        ws = self.workspace(T)
        st = _lib.moe_layer_forward_q4_host(self.shape(T), x_host, self.Wg, self.q1, self.q3, self.q2, y_host, ws,
                                            ws.numel(), stream)
        _lib.check(st, "moe_layer_forward_q4_host")

    def device_status(self, T: int) -> int:
        return _lib.moe_read_device_status(self.workspace(T))

"""Seeded synthetic inputs for the mixture-of-experts layer.

This module holds no arithmetic of the layer.  It generates the inputs that
both the GPU path (tests, ``bench.py``) and the CPU oracle consume: a
counter-based normal generator (``synth_gen.c``, definition in its header)
and the recipes of the workloads, i.e. shapes, distributions and the routing
skew, written as plain host arrays:

* ``x``   [T, d]   bfloat16 bits (uint16), ~N(0, 1)
* ``Wg``  [E, d]   float32, ~N(0, 1/d)       (router, ``nn.Linear(d, E)`` storage)
* ``W1``, ``W3`` [E, f, d] bfloat16 bits, ~N(0, 1/d)
* ``W2``  [E, d, f] bfloat16 bits, ~N(0, 1/f)

Tensor ids: x=1, Wg=2, W1=3, W3=4, W2=5.  The skewed workload sets the
constant feature x[:, 0] = 1 and adds ``SKEW_BETA`` to Wg[0, 0]; with
near-N(0,1) logits this sends about 40 % of the top-2 slots to expert 0.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth_gen.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None

TID_X, TID_WG, TID_W1, TID_W3, TID_W2 = 1, 2, 3, 4, 5
SKEW_BETA = 1.70


def build(force: bool = False) -> str:
    """Compile ``synth_gen.c`` into ``libsynth.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, i64, d = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
        lib.synth_normal_bf16.argtypes = [u64, u64, i64, d, d, ctypes.c_void_p]
        lib.synth_normal_f32.argtypes = [u64, u64, i64, d, d, ctypes.c_void_p]
        lib.synth_words.argtypes = [u64, u64, i64, ctypes.c_void_p]
        for fn in (lib.synth_normal_bf16, lib.synth_normal_f32, lib.synth_words):
            fn.restype = None
        _lib = lib
    return _lib


def normal_bf16(seed: int, tensor_id: int, shape, mean: float = 0.0, sigma: float = 1.0) -> np.ndarray:
    """bfloat16 bits (uint16 array of ``shape``) of N(mean, sigma^2) draws."""
    out = np.empty(shape, dtype=np.uint16)
    _load().synth_normal_bf16(seed, tensor_id, out.size, mean, sigma, out.ctypes.data)
    return out


def normal_f32(seed: int, tensor_id: int, shape, mean: float = 0.0, sigma: float = 1.0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    _load().synth_normal_f32(seed, tensor_id, out.size, mean, sigma, out.ctypes.data)
    return out


def words(seed: int, tensor_id: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _load().synth_words(seed, tensor_id, n, out.ctypes.data)
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bits to float32 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 bits, nearest-even (for building test inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


@dataclass
class Workload:
    """One synthetic problem: sizes, routing mode and host inputs."""
    name: str
    T: int
    d: int
    f: int
    E: int = 8
    k: int = 2
    capacity_factor: float = 0.0     # <= 0: dropless
    drop_policy: int = 0             # 0: by router probability, 1: by token order
    seed: int = 0
    skew: bool = False
    x: np.ndarray | None = field(default=None, repr=False)
    Wg: np.ndarray | None = field(default=None, repr=False)
    W1: np.ndarray | None = field(default=None, repr=False)
    W3: np.ndarray | None = field(default=None, repr=False)
    W2: np.ndarray | None = field(default=None, repr=False)

    def generate(self, weights: bool = True) -> "Workload":
        T, d, f, E, s = self.T, self.d, self.f, self.E, self.seed
        self.x = normal_bf16(s, TID_X, (T, d))
        self.Wg = normal_f32(s, TID_WG, (E, d), 0.0, 1.0 / np.sqrt(d))
        if self.skew:
            self.x[:, 0] = 0x3F80          # bf16 bits of 1.0: a constant feature
            self.Wg[0, 0] += np.float32(SKEW_BETA)
        if weights:
            self.W1 = normal_bf16(s, TID_W1, (E, f, d), 0.0, 1.0 / np.sqrt(d))
            self.W3 = normal_bf16(s, TID_W3, (E, f, d), 0.0, 1.0 / np.sqrt(d))
            self.W2 = normal_bf16(s, TID_W2, (E, d, f), 0.0, 1.0 / np.sqrt(f))
        return self

    @property
    def capacity(self) -> int | None:
        """floor(cf * T * k / E), or None when dropless."""
        if self.capacity_factor <= 0:
            return None
        return int(np.floor(np.float64(np.float32(self.capacity_factor)) * self.T * self.k / self.E))


MIXTRAL_D, MIXTRAL_F = 4096, 14336


def workload(name: str, T: int | None = None, seed: int = 0) -> Workload:
    """The named workloads: tiny, decode, prefill, skew, sweep (needs T)."""
    if name == "tiny":
        return Workload("tiny", T or 64, 128, 448, seed=seed)
    if name == "decode":
        return Workload("decode", T or 16, MIXTRAL_D, MIXTRAL_F, seed=seed)
    if name == "prefill":
        return Workload("prefill", T or 4096, MIXTRAL_D, MIXTRAL_F, seed=seed)
    if name == "skew":
        return Workload("skew", T or 8192, MIXTRAL_D, MIXTRAL_F, capacity_factor=1.25,
                        seed=seed, skew=True)
    if name == "sweep":
        if T is None:
            raise ValueError("sweep needs T")
        return Workload(f"sweep_T{T}", T, MIXTRAL_D, MIXTRAL_F, seed=seed)
    raise ValueError(f"unknown workload {name!r}")


SWEEP_T = (1, 8, 64, 512, 4096, 32768)

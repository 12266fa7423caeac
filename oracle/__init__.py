"""CPU oracle of the sparse mixture-of-experts layer (test infrastructure).

TEST INFRASTRUCTURE ONLY: the test suite, the package's smoke check and the
benchmark's CPU-baseline leg are the only callers.  The GPU path never imports
this package, and this package never imports the GPU path.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64, one function per
step of the layer, each citing the page and section it follows).  This file
only compiles it with gcc, marshals numpy arrays into it and chains the steps:

    logits -> top-k -> gates -> capacity -> grouping by expert -> experts -> y

``route(..., idx_override=...)`` re-runs the steps after top-k with indices
chosen by the caller for some tokens: the "conditional oracle" used when the
GPU picked another member of a near-tie set.  ``kept_override`` does the same
for the keep/drop decision of slots at a capacity threshold.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

DROP_BY_PROB, DROP_BY_ORDER = 0, 1
# the same policies, with a dropped slot moving to the token's next-best expert
DROP_BY_PROB_NEXT_BEST, DROP_BY_ORDER_NEXT_BEST = 2, 3


def build(force: bool = False, src: str = _SRC, out: str = _LIB, defines=()) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math", "-ffp-contract=off"]
        cmd += [f"-D{d}" for d in defines]
        subprocess.check_call(cmd + [src, "-o", tmp, "-lm"])
        os.replace(tmp, out)
    return out


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P, i64, i32, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
    sig = {
        "oracle_router_logits": [i64, i32, i32, P, P, P],
        "oracle_topk": [i64, i32, i32, P, P],
        "oracle_gates": [i64, i32, i32, P, P, P, P],
        "oracle_capacity": [i64, i32, i32, dbl, i32, P, P, P],
        "oracle_permute": [i64, i32, i32, P, P, P, P, P, P, P],
        "oracle_expert_row": [i32, i32, P, P, P, P, P, P],
        "oracle_layer_rows": [i64, i32, i32, i32, i32, P, P, P, P, P, P, P, i64, P, P, P, P],
        "oracle_num_threads": [],
        "oracle_router_stats": [i64, i32, i32, P, P, P],
        "oracle_capacity_fallback": [i64, i32, i32, dbl, i32, P, P, P, P, P, P],
        "oracle_q4_quantize": [i32, i32, i32, P, P, P],
        "oracle_q4_dequant": [i32, i32, i32, P, P, P],
        "oracle_expert_row_q4": [i32, i32, P, P, P, P, P, P, P, P, P],
        "oracle_layer_rows_q4": [i64, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P, P, i64, P, P, P,
                                 P],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = None
    lib.oracle_capacity.restype = ctypes.c_int64
    lib.oracle_capacity_fallback.restype = ctypes.c_int64
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def lib():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


class Oracle:
    """The oracle bound to one compiled library (the default build, or a
    variant compiled with extra defines, e.g. in tests that plant a mistake)."""

    def __init__(self, handle=None):
        self.L = handle if handle is not None else lib()

    @staticmethod
    def _p(a: np.ndarray):
        assert a.flags["C_CONTIGUOUS"]
        return a.ctypes.data

    def num_threads(self) -> int:
        return int(self.L.oracle_num_threads())

    def router_logits(self, x: np.ndarray, Wg: np.ndarray) -> np.ndarray:
        T, d = x.shape
        E = Wg.shape[0]
        x = np.ascontiguousarray(x, np.uint16)
        Wg = np.ascontiguousarray(Wg, np.float32)
        out = np.empty((T, E), np.float64)
        self.L.oracle_router_logits(T, d, E, self._p(x), self._p(Wg), self._p(out))
        return out

    def topk(self, logits: np.ndarray, k: int) -> np.ndarray:
        logits = np.ascontiguousarray(logits, np.float64)
        T, E = logits.shape
        idx = np.empty((T, k), np.int32)
        self.L.oracle_topk(T, E, k, self._p(logits), self._p(idx))
        return idx

    def gates(self, logits: np.ndarray, idx: np.ndarray):
        logits = np.ascontiguousarray(logits, np.float64)
        idx = np.ascontiguousarray(idx, np.int32)
        T, E = logits.shape
        k = idx.shape[1]
        w = np.empty((T, k), np.float64)
        p = np.empty((T, k), np.float64)
        self.L.oracle_gates(T, E, k, self._p(logits), self._p(idx), self._p(w), self._p(p))
        return w, p

    def capacity(self, idx: np.ndarray, p: np.ndarray, E: int, cf: float, policy: int):
        idx = np.ascontiguousarray(idx, np.int32)
        p = np.ascontiguousarray(p, np.float64)
        T, k = idx.shape
        kept = np.empty(T * k, np.uint8)
        cap = self.L.oracle_capacity(T, E, k, float(cf), int(policy), self._p(idx), self._p(p),
                                     self._p(kept))
        return kept, (None if cap < 0 else int(cap))

    def capacity_fallback(self, logits: np.ndarray, idx: np.ndarray, p: np.ndarray, E: int, cf: float,
                          policy: int, order_override=None):
        """Capacity with the next-best-expert fallback (policy 0 / 1 as in
        capacity()).  order_override: (T, E) int array or None; a row whose
        first entry is >= 0 replaces that token's router order.  Returns
        (expert per slot, kept, cap)."""
        logits = np.ascontiguousarray(logits, np.float64)
        idx = np.ascontiguousarray(idx, np.int32)
        p = np.ascontiguousarray(p, np.float64)
        T, k = idx.shape
        expert = np.empty(T * k, np.int32)
        kept = np.empty(T * k, np.uint8)
        ov = None if order_override is None else np.ascontiguousarray(order_override, np.int32)
        cap = self.L.oracle_capacity_fallback(T, E, k, float(cf), int(policy), self._p(logits), self._p(idx),
                                              self._p(p), self._p(ov) if ov is not None else None,
                                              self._p(expert), self._p(kept))
        return expert, kept, (None if cap < 0 else int(cap))

    def permute(self, idx: np.ndarray, kept: np.ndarray, E: int):
        idx = np.ascontiguousarray(idx, np.int32)
        kept = np.ascontiguousarray(kept, np.uint8)
        T, k = idx.shape
        S = T * k
        counts = np.empty(E, np.int32)
        kept_counts = np.empty(E, np.int32)
        offsets = np.empty(E + 1, np.int32)
        perm_slot = np.full(max(S, 1), -1, np.int32)
        slot_pos = np.empty(max(S, 1), np.int32)
        self.L.oracle_permute(T, E, k, self._p(idx), self._p(kept), self._p(counts),
                              self._p(kept_counts), self._p(offsets), self._p(perm_slot),
                              self._p(slot_pos))
        n = int(offsets[E])
        return dict(counts=counts, kept_counts=kept_counts, offsets=offsets,
                    perm_slot=perm_slot[:n], slot_pos=slot_pos[:S])

    def expert_row(self, xrow, W1e, W3e, W2e):
        f, d = W1e.shape
        xrow = np.ascontiguousarray(xrow, np.uint16)
        W1e, W3e, W2e = (np.ascontiguousarray(a, np.uint16) for a in (W1e, W3e, W2e))
        h = np.empty(f, np.float64)
        o = np.empty(d, np.float64)
        self.L.oracle_expert_row(d, f, self._p(xrow), self._p(W1e), self._p(W3e), self._p(W2e),
                                 self._p(h), self._p(o))
        return h, o

    def route(self, x, Wg, k: int, cf: float = 0.0, policy: int = DROP_BY_PROB,
              idx_override=None, kept_override=None, logits=None, order_override=None) -> dict:
        """Steps logits .. grouping.  ``idx_override``: (T, k) array or None;
        entries >= 0 replace the oracle's top-k choice for that token (all k
        of a row are replaced together).  ``kept_override``: (S,) int array or
        None; entries >= 0 replace the keep/drop decision of that slot."""
        E = Wg.shape[0]
        if logits is None:
            logits = self.router_logits(x, Wg)
        idx = self.topk(logits, k)
        if idx_override is not None:
            rows = np.all(idx_override >= 0, axis=1)
            idx = idx.copy()
            idx[rows] = idx_override[rows]
        w, p = self.gates(logits, idx)
        if policy >= DROP_BY_PROB_NEXT_BEST:
            assert kept_override is None
            expert, kept, cap = self.capacity_fallback(logits, idx, p, E, cf, policy - 2, order_override)
            perm = self.permute(expert.reshape(idx.shape), kept, E)
            # counts stay the router's histogram; the grouping follows `expert`
            perm["counts"] = np.bincount(idx.ravel(), minlength=E).astype(np.int32)
            return dict(logits=logits, idx=idx, w=w, p=p, kept=kept, cap=cap, expert=expert.reshape(idx.shape),
                        **perm)
        kept, cap = self.capacity(idx, p, E, cf, policy)
        if kept_override is not None:
            sel = kept_override >= 0
            kept = kept.copy()
            kept[sel] = kept_override[sel].astype(np.uint8)
        perm = self.permute(idx, kept, E)
        return dict(logits=logits, idx=idx, w=w, p=p, kept=kept, cap=cap, expert=idx, **perm)

    def layer_rows(self, x, W1, W3, W2, route: dict, rows, want_h: bool = False,
                   want_o: bool = False):
        """y (fp64) for the token indices in ``rows``; optionally per-slot h and o."""
        T, d = x.shape
        E, f, _ = W1.shape
        idx, w, kept = route.get("expert", route["idx"]), route["w"], route["kept"]
        k = idx.shape[1]
        rows = np.ascontiguousarray(rows, np.int64)
        n = rows.shape[0]
        y = np.empty((n, d), np.float64)
        h = np.empty((n, k, f), np.float64) if want_h else None
        o = np.empty((n, k, d), np.float64) if want_o else None
        args = [np.ascontiguousarray(a, np.uint16) for a in (x, W1, W3, W2)]
        idx = np.ascontiguousarray(idx, np.int32)
        w = np.ascontiguousarray(w, np.float64)
        kept = np.ascontiguousarray(kept, np.uint8)
        self.L.oracle_layer_rows(T, d, f, E, k, *(self._p(a) for a in args), self._p(idx),
                                 self._p(w), self._p(kept), n, self._p(rows), self._p(y),
                                 self._p(h) if h is not None else None,
                                 self._p(o) if o is not None else None)
        out = dict(y=y)
        if want_h:
            out["h"] = h
        if want_o:
            out["o"] = o
        return out

    def router_stats(self, idx: np.ndarray, E: int):
        """Per-slot expert histograms [k, E] and first-two-choice pair counts
        [E, E] of top-k indices idx [T, k]."""
        idx = np.ascontiguousarray(idx, np.int32)
        T, k = idx.shape
        slot = np.empty((k, E), np.int32)
        pair = np.empty((E, E), np.int32)
        self.L.oracle_router_stats(T, E, k, self._p(idx), self._p(slot), self._p(pair))
        return slot, pair

    # ------------------------------------------------------------ 4-bit experts
    def q4_quantize(self, W: np.ndarray):
        """W [E, R, K] bf16 bits -> (codes [E, R, K/2] uint8, scales [E, K/64, R]
        bf16 bits): symmetric 4-bit codes with one absmax scale per 64 inputs."""
        W = np.ascontiguousarray(W, np.uint16)
        E, R, K = W.shape
        assert K % 64 == 0
        codes = np.empty((E, R, K // 2), np.uint8)
        scales = np.empty((E, K // 64, R), np.uint16)
        self.L.oracle_q4_quantize(E, R, K, self._p(W), self._p(codes), self._p(scales))
        return codes, scales

    def q4_dequant(self, codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
        """(codes, scales) -> w_hat [E, R, K] in fp64."""
        codes = np.ascontiguousarray(codes, np.uint8)
        scales = np.ascontiguousarray(scales, np.uint16)
        E, R, K2 = codes.shape
        out = np.empty((E, R, 2 * K2), np.float64)
        self.L.oracle_q4_dequant(E, R, 2 * K2, self._p(codes), self._p(scales), self._p(out))
        return out

    def layer_rows_q4(self, x, q1, q3, q2, route: dict, rows, want_h: bool = False,
                      want_o: bool = False):
        """layer_rows with 4-bit expert weights; q1, q3, q2 are the (codes,
        scales) pairs of W1, W3 [E, f, d] and W2 [E, d, f]."""
        T, d = x.shape
        E, f, _ = q1[0].shape
        idx, w, kept = route.get("expert", route["idx"]), route["w"], route["kept"]
        k = idx.shape[1]
        rows = np.ascontiguousarray(rows, np.int64)
        n = rows.shape[0]
        y = np.empty((n, d), np.float64)
        h = np.empty((n, k, f), np.float64) if want_h else None
        o = np.empty((n, k, d), np.float64) if want_o else None
        x = np.ascontiguousarray(x, np.uint16)
        ws = []
        for c, sc in (q1, q3, q2):
            ws += [np.ascontiguousarray(c, np.uint8), np.ascontiguousarray(sc, np.uint16)]
        idx = np.ascontiguousarray(idx, np.int32)
        w = np.ascontiguousarray(w, np.float64)
        kept = np.ascontiguousarray(kept, np.uint8)
        self.L.oracle_layer_rows_q4(T, d, f, E, k, self._p(x), *(self._p(a) for a in ws), self._p(idx),
                                    self._p(w), self._p(kept), n, self._p(rows), self._p(y),
                                    self._p(h) if h is not None else None,
                                    self._p(o) if o is not None else None)
        out = dict(y=y)
        if want_h:
            out["h"] = h
        if want_o:
            out["o"] = o
        return out

    def layer(self, x, Wg, W1, W3, W2, k: int, cf: float = 0.0, policy: int = DROP_BY_PROB):
        r = self.route(x, Wg, k, cf, policy)
        r.update(self.layer_rows(x, W1, W3, W2, r, np.arange(x.shape[0])))
        return r


def default() -> Oracle:
    return Oracle()

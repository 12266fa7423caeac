"""Run the MoE layer on one synthetic shape and print its step time.

    python -m sparse_mixture_experts_13_b200.run_case --T 1024 --E 2 --iters 5

Inputs come from the seeded generator (x ~ N(0,1), Wg ~ N(0,1/d),
W1/W3 ~ N(0,1/d), W2 ~ N(0,1/f)).  Useful for profiling reduced cases of the
benchmark's workloads.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

from . import _lib  # noqa: E402
from .layer import MoELayer, MoELayerQ4  # noqa: E402


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--T", type=int, default=4096)
    ap.add_argument("--d", type=int, default=4096)
    ap.add_argument("--f", type=int, default=14336)
    ap.add_argument("--E", type=int, default=8)
    ap.add_argument("--k", type=int, default=2)
    ap.add_argument("--cf", type=float, default=0.0)
    ap.add_argument("--policy", type=int, default=0)
    ap.add_argument("--variant", type=int, default=0)
    ap.add_argument("--skew", action="store_true")
    ap.add_argument("--q4", action="store_true", help="4-bit expert weights (quantised on the device)")
    ap.add_argument("--iters", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=1)
    a = ap.parse_args(argv)
    wl = synth.Workload("case", a.T, a.d, a.f, E=a.E, k=a.k, capacity_factor=a.cf, drop_policy=a.policy,
                        skew=a.skew).generate()
    dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).cuda()
    if a.q4:
        layer = MoELayerQ4.from_bf16(torch.from_numpy(wl.Wg).cuda(), dev(wl.W1), dev(wl.W3), dev(wl.W2), k=a.k,
                                     capacity_factor=a.cf, drop_policy=a.policy)
    else:
        layer = MoELayer(torch.from_numpy(wl.Wg).cuda(), dev(wl.W1), dev(wl.W3), dev(wl.W2), k=a.k,
                         capacity_factor=a.cf, drop_policy=a.policy, gemm_variant=a.variant)
    x = dev(wl.x)
    y = torch.empty(a.T, a.d, dtype=torch.bfloat16, device="cuda")
    for _ in range(a.warmup):
        layer.forward(x, y)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(a.iters):
        layer.forward(x, y)
    e.record()
    torch.cuda.synchronize()
    st = layer.device_status(a.T)
    _lib.check(st, "device status")
    ms = s.elapsed_time(e) / max(1, a.iters)
    flops = 6.0 * a.T * a.k * a.d * a.f + 2.0 * a.T * a.d * a.E
    print(f"T={a.T} d={a.d} f={a.f} E={a.E} k={a.k} cf={a.cf} variant={a.variant} q4={a.q4}: {ms:.4f} ms/step, "
          f"{a.T / ms * 1e3:.1f} tokens/s, {flops / ms / 1e9:.1f} TFLOP/s (dropless count)")


if __name__ == "__main__":
    main()

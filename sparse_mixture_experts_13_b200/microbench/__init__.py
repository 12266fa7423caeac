"""Microbenchmarks behind kernel design choices (not part of the layer).

``python -m sparse_mixture_experts_13_b200.microbench`` builds and runs
``mma_issue.cu``: the issue cost of tcgen05.mma kind::f16 against kind::i8
at the small N of the decode GEMMs, one JSON line per configuration.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def build() -> str:
    out = os.path.join(PKG, "_build", "mma_issue")
    os.makedirs(os.path.dirname(out), exist_ok=True)
    src = os.path.join(HERE, "mma_issue.cu")
    hdr = os.path.join(PKG, "csrc", "sm100.cuh")
    if not os.path.exists(out) or max(os.path.getmtime(src), os.path.getmtime(hdr)) > os.path.getmtime(out):
        subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
                        f"-I{os.path.join(PKG, 'csrc')}", src, "-o", out], check=True)
    return out


def main(argv=None) -> int:
    exe = build()
    return subprocess.run([exe] + list(argv if argv is not None else sys.argv[1:])).returncode


if __name__ == "__main__":
    sys.exit(main())

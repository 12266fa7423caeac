"""Build ``libmoe.so`` (the C ABI of include/moe.h) for sm_100a with nvcc.

Objects go to ``_build/`` beside this file; the shared library is written
in-tree so that it travels with the source tree.  Rebuilds only what changed.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libmoe.so")
# debug build: -DMOE_DEBUG (device-side bounds checks, workspace guards,
# stage-failure hook), objects in _build/debug
LIB_DEBUG = os.path.join(PKG, "libmoe_debug.so")
SOURCES = ["router.cu", "permute.cu", "expert_gemm.cu", "expert_gemm_q4.cu", "expert_gemm_q4i8.cu", "router_stats.cu", "fallback.cu", "ep.cu", "combine.cu", "moe_api.cu", "selftest.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
                "--expt-relaxed-constexpr", f"-I{INCLUDE}", f"-I{CSRC}"]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, extra, outdir=BUILD):
    obj = os.path.join(outdir, os.path.basename(src).replace(".cu", ".o"))
    if _stale(obj, [src] + _headers()):
        cmd = [NVCC] + FLAGS + list(extra) + ["-c", src, "-o", obj]
        subprocess.run(cmd, check=True)
    return obj


def build(force: bool = False, extra_flags=(), verbose_ptxas: bool = False, debug: bool = False) -> str:
    outdir = os.path.join(BUILD, "debug") if debug else BUILD
    lib = LIB_DEBUG if debug else LIB
    os.makedirs(outdir, exist_ok=True)
    extra = list(extra_flags) + (["-Xptxas", "-v"] if verbose_ptxas else []) + (["-DMOE_DEBUG"] if debug else [])
    if force:
        for o in glob.glob(os.path.join(outdir, "*.o")):
            os.remove(o)
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    with cf.ThreadPoolExecutor(max_workers=len(srcs)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, outdir), srcs))
    if force or _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.run([NVCC] + ARCH + ["-shared", "-o", tmp] + objs, check=True)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    import sys
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv, debug="--debug" in sys.argv))

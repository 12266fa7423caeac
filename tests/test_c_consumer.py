"""The boundary from plain C: a C99 program includes include/moe.h, links
libmoe.so and calls the entry points that need no GPU (sizes, status text,
argument checks), so the header is valid C and the exported symbols resolve
through an ordinary link, not only through ctypes."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "moe.h"

int main(void) {
  moe_shape sh = {4096, 4096, 14336, 8, 2, 0.0f, MOE_DROP_BY_PROB, MOE_VARIANT_AUTO};
  size_t n = moe_workspace_size(&sh);
  moe_shape q = sh;
  q.T = 16;
  size_t nq = moe_workspace_size_q4(&q);
  moe_shape bad = sh;
  bad.k = 9;                                   /* k > 8: invalid */
  if (moe_workspace_size(&bad) != 0) return 2;
  /* invalid shape: rejected before any device work */
  moe_status st = moe_layer_forward(&bad, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL);
  if (st != MOE_ERR_INVALID_ARG) return 3;
  /* T == 0 is a no-op */
  moe_shape empty = sh;
  empty.T = 0;
  if (moe_combine(&empty, NULL, NULL, NULL, NULL, NULL) != MOE_OK) return 4;
  if (strcmp(moe_status_string(MOE_ERR_TIMEOUT), "device-side wait timed out") != 0) return 5;
  printf("%zu %zu\n", n, nq);
  return 0;
}
"""


@pytest.fixture(scope="module")
def lib_path():
    from sparse_mixture_experts_13_b200 import build as b
    return b.build()


def test_c_program_links_and_runs(lib_path):
    import sparse_mixture_experts_13_b200 as moe
    tmp = tempfile.mkdtemp(prefix="moe_c_")
    src = os.path.join(tmp, "consumer.c")
    exe = os.path.join(tmp, "consumer")
    with open(src, "w") as fh:
        fh.write(PROGRAM)
    libdir = os.path.dirname(lib_path)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src, "-o", exe,
                    "-L", libdir, "-lmoe", f"-Wl,-rpath,{libdir}"], check=True, capture_output=True, text=True)
    try:
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    n, nq = map(int, r.stdout.split())
    assert n == moe.moe_workspace_size(moe.make_shape(4096, 4096, 14336))
    assert nq == moe.moe_workspace_size_q4(moe.make_shape(16, 4096, 14336))

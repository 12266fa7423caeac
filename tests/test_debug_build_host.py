"""The debug build of the library (libmoe_debug.so, compiled with MOE_DEBUG)
on a host without a GPU: it loads, reports itself as the debug build, exports
the same symbols as the header, and its workspaces are larger than the
release build's by one 256-byte guard per region past the control region.
The release build reports 0 and refuses the guard calls."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_PROBE = r"""
import json, sys
sys.path.insert(0, {root!r})
import sparse_mixture_experts_13_b200 as moe
sizes = {{}}
for name, args in dict(pair=(300, 128, 448, 8, 2, 0.0, 0, 1), stream=(16, 4096, 14336, 8, 2, 0.0, 0, 2),
                       fallback=(1000, 128, 256, 8, 2, 1.25, 2, 1)).items():
    sizes[name] = [moe.moe_workspace_size(moe.make_shape(*args)), moe.moe_workspace_size_q4(moe.make_shape(*args))]
sh = moe.make_shape(64, 128, 448)
print(json.dumps(dict(lib=moe._lib.LIB_PATH, debug=moe.moe_debug_build(), sizes=sizes,
                      arm=moe.moe_debug_workspace_arm(sh, 1 << 20, 1 << 30, False, 0),
                      bounds=moe.MOE_ERR_BOUNDS, text=moe.status_string(moe.MOE_ERR_BOUNDS))))
"""


def _probe(lib):
    from sparse_mixture_experts_13_b200 import build as b
    b.build(debug=(lib == "debug"))
    env = dict(os.environ, MOE_LIB=lib)
    r = subprocess.run([sys.executable, "-c", _PROBE.format(root=ROOT)], capture_output=True, text=True,
                       timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


@pytest.fixture(scope="module")
def both():
    return _probe("release"), _probe("debug")


def test_debug_library_identifies_itself(both):
    rel, dbg = both
    assert rel["lib"].endswith("libmoe.so") and dbg["lib"].endswith("libmoe_debug.so")
    assert rel["debug"] == 0 and dbg["debug"] == 1
    assert rel["arm"] == 2                      # MOE_ERR_UNSUPPORTED in the release build
    assert dbg["bounds"] == 6 and "bounds" in dbg["text"]


def test_debug_workspaces_carry_guards(both):
    rel, dbg = both
    for name in rel["sizes"]:
        for r, d in zip(rel["sizes"][name], dbg["sizes"][name]):
            extra = d - r
            # one 256-byte guard after each region past the control region
            assert extra > 0 and extra % 256 == 0 and 12 <= extra // 256 <= 32, (name, r, d)

"""The debug build (libmoe_debug.so: device-side bounds checks, workspace
guards, stage-failure hook), exercised in a child process with MOE_LIB=debug:

* the small-size parity cases of test_gpu_parity.py, every layer and stage
  call with its workspace guards armed before and checked after (see
  gpu_harness.guarded), outputs against the oracle as in the release run;
* debug_hooks_cases.py: the stage-failure hook and the bounds checks.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

SMALL = ("tiny or capacity_many or expert_counts or ragged or noop or hot5 or exact_logit or zero_input "
         "or capacity_zero or variants_agree or router_many")


def test_debug_build_under_guards():
    from sparse_mixture_experts_13_b200 import build as b
    b.build(debug=True)
    env = dict(os.environ, MOE_LIB="debug")
    env.pop("MOE_DEBUG_FAIL_STAGE", None)
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
           os.path.join(HERE, "test_gpu_parity.py"), "-k", SMALL, os.path.join(HERE, "debug_hooks_cases.py")]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=1500, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and " failed" not in r.stdout

"""The expert-parallel bench arm (bench.py --ep) on one GPU: one rank owns
all experts, so every row stays local; the line must be well formed and the
step must finish."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_bench_ep_one_rank():
    env = dict(os.environ)
    for v in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_PORT"):
        env.pop(v, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--ep", "--gpus", "1", "--steps", "2",
                        "--warmup", "3", "--ep-tokens", "256"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert line["n_gpus"] == 1 and line["config"]["parallelism"] == "ep1"
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert set(line["phases_ms"]) == {"route_and_plan", "dispatch", "expert_gemms", "combine"}
    assert line["dispatch"]["bytes_per_rank"] == 0 and line["return"]["bytes_per_rank"] == 0

"""Host logic of bench.py that needs no GPU: the clock samples taken during
the timed region, the DRAM-traffic record that is reported only while the
kernel sources are unchanged since the capture, and the warm-up floor."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


class _Done:
    def terminate(self):
        pass

    def wait(self):
        return 0


def _sampler_with(rows, pci):
    s = bench.ClockSampler(pci)
    s.file.write("\n".join(rows) + "\n")
    s.proc = _Done()
    return s


def _row(bus, sm, mx, power, reasons=("Not Active",) * 4):
    return ", ".join(["0", bus, str(sm), str(mx), str(power), "0x0"] + list(reasons))


def test_clock_samples_of_this_gpu_only():
    mine, other = "00000000:1B:00.0", "00000000:2C:00.0"
    rows = [_row(mine, 1900, 1965, 700), _row(other, 600, 1965, 100, ("Active",) * 4),
            _row(mine, 1300, 1965, 998, ("Not Active", "Not Active", "Not Active", "Active")),
            _row(mine, 1500, 1965, 900)]
    c = _sampler_with(rows, "00000000:1b:00.0").stop()
    assert c["samples"] == 3
    assert c["sm_mhz"] == 1500 and c["sm_max_mhz"] == 1965 and c["power_w_max"] == 998
    assert c["reasons"] == ["sw_power_cap"]        # the other GPU's slowdowns are not ours


def test_clock_reasons_reported():
    bus = "00000000:1B:00.0"
    rows = [_row(bus, 1200, 1965, 1000, ("Active", "Not Active", "Active", "Not Active"))]
    c = _sampler_with(rows, None).stop()
    assert c["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_sampler_without_nvidia_smi():
    s = bench.ClockSampler(None)
    s.proc = None
    c = s.stop()
    s.file.close()
    os.unlink(s.file.name)
    assert c["sm_mhz"] is None and c["samples"] == 0


def _fake_tree(tmp, src_text):
    csrc = tmp / "sparse_mixture_experts_13_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(src_text)
    (tmp / "profiles").mkdir()
    return bench.kernel_source_sha(str(tmp))


def test_strip_c_comments():
    src = ('#include "a.h"  // the header\n/* block\n comment */ int f(char c) {\n'
           '  const char* s = "not // a comment /* either */";\n  return c == \'"\' ? 1 : \'/\';  // done\n}\n')
    assert bench.strip_c_comments(src) == ('#include "a.h" int f(char c) { const char* s = '
                                           '"not // a comment /* either */"; return c == \'"\' ? 1 : \'/\'; }')


def test_traffic_record_only_for_unchanged_kernels(tmp_path, monkeypatch):
    code = "// kernel k\n__global__ void k(int* p) { p[0] = 1; }\n"
    sha = _fake_tree(tmp_path, code)
    rec = [dict(kernel="k", workload="w", source_sha=sha, dram_bytes_per_launch=1234)]
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    cu = tmp_path / "sparse_mixture_experts_13_b200" / "csrc" / "k.cu"
    assert bench.traffic_record("k", "w") == 1234
    assert bench.traffic_record("k", "other") is None
    cu.write_text("/* kernel k, reworded\n   over two lines */\n__global__ void k(int* p) {\n  p[0] = 1;\n}\n")
    assert bench.traffic_record("k", "w") == 1234   # comments and layout only
    cu.write_text(code.replace("p[0] = 1", "p[0] = 2"))
    assert bench.traffic_record("k", "w") is None   # the kernel changed since the capture


def test_traffic_record_missing_file(tmp_path, monkeypatch):
    _fake_tree(tmp_path, "x")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("k", "w") is None


def test_warmup_floor():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2", "--steps", "1"],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "warmup" in r.stderr


@pytest.mark.parametrize("d,f", [(4096, 14336), (128, 448)])
def test_expert_bytes(d, f):
    assert bench.expert_bytes(d, f) == 3 * d * f * 2
    # 4 bits a weight plus one bf16 scale per 64 weights
    assert bench.expert_bytes_q4(d, f) * 64 == 3 * d * f * (32 + 2)

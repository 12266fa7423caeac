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


def test_traffic_record_scoped_to_its_files(tmp_path, monkeypatch):
    code = "__global__ void k(int* p) { p[0] = 1; }\n"
    _fake_tree(tmp_path, code)
    csrc = tmp_path / "sparse_mixture_experts_13_b200" / "csrc"
    (csrc / "other.cu").write_text("__global__ void o(int* p) { p[0] = 3; }\n")
    sha = bench.kernel_source_sha(str(tmp_path), ["k.cu"])
    assert sha != bench.kernel_source_sha(str(tmp_path))
    rec = [dict(kernel="k", workload="w", source_sha=sha, source_files=["k.cu"], dram_bytes_per_launch=77)]
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("k", "w") == 77
    (csrc / "other.cu").write_text("__global__ void o(int* p) { p[0] = 4; }\n")
    assert bench.traffic_record("k", "w") == 77     # a file the kernel is not built from changed
    (csrc / "k.cu").write_text(code.replace("p[0] = 1", "p[0] = 2"))
    assert bench.traffic_record("k", "w") is None   # its own source changed
    (csrc / "k.cu").unlink()
    assert bench.traffic_record("k", "w") is None   # or went away


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


class _FakeNvml:
    """Just the NVML calls NvmlSampler makes, over a scripted clock trace."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonHwPowerBrakeSlowdown = 0x80

    class _Pci:
        def __init__(self, bus):
            self.busId = bus

    def __init__(self, buses, trace):
        self.buses, self.trace, self.i = buses, trace, 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetCount(self):
        return len(self.buses)

    def nvmlDeviceGetHandleByIndex(self, i):
        return i

    def nvmlDeviceGetPciInfo(self, h):
        return self._Pci(self.buses[h].encode())

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        assert h == 1, "sampled the wrong GPU"
        return self.trace[min(self.i, len(self.trace) - 1)][0]

    def nvmlDeviceGetPowerUsage(self, h):
        return self.trace[min(self.i, len(self.trace) - 1)][1] * 1000

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        r = self.trace[min(self.i, len(self.trace) - 1)][2]
        self.i += 1
        return r


def test_nvml_sampler_regions_and_reasons():
    fake = _FakeNvml(["00000000:1A:00.0", "00000000:1B:00.0"],
                     [(1965, 300, 0), (1900, 500, 0), (1500, 990, 0x4), (1300, 1000, 0x4 | 0x20)])
    s = bench.NvmlSampler("00000000:1b:00.0", nvml=fake)   # picks device 1 by PCI bus id
    assert s.max_mhz == 1965
    s.sample("decode")
    s.sample("decode")
    s.sample("prefill")
    s.sample("prefill")
    c = s.stop()
    assert c["samples"] == 4 and c["sm_max_mhz"] == 1965
    assert c["by_region"]["decode"]["sm_mhz"] == 1932.5 and c["by_region"]["decode"]["reasons"] == []
    assert c["by_region"]["prefill"]["sm_mhz"] == 1400 and c["by_region"]["prefill"]["power_w_max"] == 1000
    assert c["by_region"]["prefill"]["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
    assert c["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]


def test_nvml_sampler_samples_only_inside_regions():
    import time as _t
    fake = _FakeNvml(["00000000:1A:00.0", "00000000:1B:00.0"], [(1965, 300, 0)])
    s = bench.NvmlSampler("00000000:1B:00.0", period_s=0.001, nvml=fake)
    s.start()
    _t.sleep(0.02)
    assert s.samples == []
    with s.region("prefill"):
        _t.sleep(0.05)
    n = len(s.samples)
    _t.sleep(0.02)
    c = s.stop()
    assert n > 0 and len(s.samples) <= n + 1
    assert set(c["by_region"]) == {"prefill"}


def test_dry_run_launches_ranks():
    """--gpus 2 without torchrun relaunches itself with two ranks; the slower
    rank's step time (2 ms) is reported and the value counts both ranks."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1])
    assert line["n_gpus"] == 2 and line["ranks_seen"] == 2
    assert line["ms_per_step"] == 2.0 and line["value"] == 2 * 4096 / 2e-3


def test_world_size_must_match_gpus():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run", "--warmup", "3"],
                       capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode != 0 and "--gpus 2 but 1 ranks" in r.stderr


def test_both_arms_share_the_config():
    import synth
    wl = synth.workload("prefill")
    assert bench.bench_config(wl, 1) == bench.bench_config(synth.workload("prefill"), 1)
    assert bench.bench_config(wl, 8)["parallelism"].startswith("dp8")

"""Benchmark of the sparse MoE layer on B200: one JSON line on rank 0.

A step is one whole forward of the layer (router, top-2 gate, grouping by
expert, grouped SwiGLU expert GEMMs, combine) over one batch of synthetic
Mixtral-shaped input (d_model 4096, d_ff 14336, 8 experts, top-2, seed 0
weights; every rank draws its own tokens).  The headline workload is prefill,
T = 4096 tokens, on the tensor-core roofline; the decode workload, T = 16, is
reported beside it on the HBM roofline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU runs (one rank per GPU) shard the tokens: each rank runs the same
layer on its own batch with no data-path collective (weak scaling); the step
time is the max over ranks.  Under torchrun the ranks come from the
environment; ``--gpus N`` with N > 1 and no WORLD_SIZE relaunches this script
under torchrun with N ranks.  ``--impl reference`` times the CPU oracle on the
host cores on a bounded sample of the same workload.  ``--dry-run`` checks the
launcher and the rank plumbing without a GPU (gloo, a fixed step time per
rank).

Clocks are sampled in-process through NVML (read-only queries) every 5 ms
while a timed loop runs, per workload.
"""
from __future__ import annotations

import argparse
import contextlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s; % bf16 TC peak (T=4096) and % HBM BW (T=16)"
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            pk = json.load(fh)
        return dict(hbm=float(pk["hbm_gbs"]), bf16=float(pk["bf16_tflops"]),
                    bf16_sustained=float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS, bf16_sustained=FALLBACK_BF16_TFLOPS,
                    source="fallback")


def strip_c_comments(text: str) -> str:
    """C/C++/CUDA source without its comments, whitespace runs collapsed to
    one space: what the compiler sees, so that editing a comment does not
    count as changing a kernel."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_sha(root: str = None, files=None) -> str:
    """Hash of the CUDA sources (comments and layout ignored): the named
    files of the source folder, else all of them."""
    import hashlib
    src = os.path.join(root or ROOT, "sparse_mixture_experts_13_b200", "csrc")
    h = hashlib.sha256()
    names = sorted(files) if files else sorted(os.listdir(src))
    for name in names:
        if name.endswith((".cu", ".cuh", ".h")):
            try:
                with open(os.path.join(src, name), encoding="utf-8") as fh:
                    h.update(strip_c_comments(fh.read()).encode())
            except OSError:
                h.update(b"\0missing:" + name.encode())
    return h.hexdigest()[:16]


def traffic_record(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, only while the
    kernel sources are unchanged (up to comments) since the capture (else
    None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as fh:
            recs = json.load(fh)
    except (OSError, ValueError):
        return None
    for r in recs:
        if r.get("kernel") != kernel or r.get("workload") != workload:
            continue
        # a record names the files its kernel is built from; the others may change
        if r.get("source_sha") == kernel_source_sha(ROOT, r.get("source_files")):
            return r.get("dram_bytes_per_launch")
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU is busy."""
    QUERY = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, pci_bus_id: str | None):
        self.pci = (pci_bus_id or "").lower()
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"], samples=0)
        self.proc.terminate()
        self.proc.wait()
        self.file.flush()
        self.file.seek(0)
        rows = [list(map(str.strip, ln.split(","))) for ln in self.file.read().splitlines() if ln.strip()]
        os.unlink(self.file.name)
        bus = {r[1].lower() for r in rows}
        if len(bus) > 1 and self.pci:
            rows = [r for r in rows if r[1].lower().endswith(self.pci[-12:])]
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        power = [float(r[4]) for r in rows if r[4].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[6:10]) if v.strip().lower() == "active"})
        return dict(sm_mhz=statistics.median(sm) if sm else None, sm_max_mhz=max(mx) if mx else None,
                    power_w_max=max(power) if power else None, reasons=reasons, samples=len(sm))


class NvmlSampler:
    """This GPU's SM clock, power draw and clock-event reasons, queried
    in-process through NVML (read-only) every `period_s` while a timed region
    is open.  Samples are tagged with the region's name; nothing is sampled
    outside regions, so every sample is "under load"."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, pci_bus_id: str | None, period_s: float = 0.005, nvml=None):
        if nvml is None:
            import pynvml as nvml
        self.nvml = nvml
        nvml.nvmlInit()
        self.handle = self._find(pci_bus_id)
        self.max_mhz = float(nvml.nvmlDeviceGetMaxClockInfo(self.handle, nvml.NVML_CLOCK_SM))
        self.masks = [(name, int(getattr(nvml, attr, 0))) for name, attr in self.REASONS]
        self.period = period_s
        self.samples = []          # (tag, sm_mhz, power_w, reason mask)
        self._tag = None
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._run, daemon=True)

    def _find(self, pci):
        nv = self.nvml
        n = nv.nvmlDeviceGetCount()
        want = (pci or "").lower()[-12:]
        for i in range(n):
            h = nv.nvmlDeviceGetHandleByIndex(i)
            bus = nv.nvmlDeviceGetPciInfo(h).busId
            bus = bus.decode() if isinstance(bus, bytes) else str(bus)
            if want and bus.lower().endswith(want):
                return h
        if n == 1 or not want:
            return nv.nvmlDeviceGetHandleByIndex(0)
        raise RuntimeError(f"no NVML device with PCI bus id {pci}")

    def _reasons(self):
        nv = self.nvml
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(fn(self.handle))

    def sample(self, tag):
        nv = self.nvml
        sm = float(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
        pw = float(nv.nvmlDeviceGetPowerUsage(self.handle)) / 1000.0
        self.samples.append((tag, sm, pw, self._reasons()))

    def _run(self):
        while not self._stop.is_set():
            tag = self._tag
            if tag is not None:
                try:
                    self.sample(tag)
                except Exception:  # a failed query leaves no sample
                    pass
            self._stop.wait(self.period)

    def start(self):
        self._thread.start()

    @contextlib.contextmanager
    def region(self, tag: str):
        self._tag = tag
        try:
            yield
        finally:
            self._tag = None

    def _summary(self, rows) -> dict:
        sm = [r[1] for r in rows]
        reasons = sorted({n for r in rows for n, m in self.masks if m and (r[3] & m)})
        return dict(sm_mhz=statistics.median(sm) if sm else None, sm_max_mhz=self.max_mhz,
                    power_w_max=max((r[2] for r in rows), default=None), reasons=reasons, samples=len(rows))

    def stop(self) -> dict:
        self._stop.set()
        if self._thread.is_alive():
            self._thread.join(timeout=1.0)
        out = self._summary(self.samples)
        out["source"] = f"NVML, every {self.period * 1e3:.0f} ms inside the timed loops"
        tags = []
        for r in self.samples:
            if r[0] not in tags:
                tags.append(r[0])
        out["by_region"] = {t: self._summary([r for r in self.samples if r[0] == t]) for t in tags}
        return out


def make_clock_sampler(pci):
    """NVML in-process sampler, else nvidia-smi polling."""
    try:
        return NvmlSampler(pci)
    except Exception:
        return ClockSampler(pci)


def sampler_region(sampler, tag):
    return sampler.region(tag) if hasattr(sampler, "region") else contextlib.nullcontext()


# ---------------------------------------------------------------- helpers

def to_dev_bf16(a, torch):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def max_over_ranks(value: float, torch, dist=None, device="cuda") -> float:
    """The largest `value` over all ranks (every rank gets it)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch per step."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def time_steps(fn, steps, torch, dist=None):
    """K steps between a barrier + synchronize on both sides; CUDA events on
    the current stream; max over ranks."""
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        fn()
    end.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    return max_over_ranks(start.elapsed_time(end), torch, dist)


def flushed_median_ms(fn, iters, torch, flush, dist=None):
    """Median of per-iteration CUDA-event times, L2 flushed before every
    iteration by writing `flush` (a buffer over twice the L2 size); max over
    ranks of each rank's median."""
    times = []
    torch.cuda.synchronize()
    for i in range(iters):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    return max_over_ranks(statistics.median(times), torch, dist)


class Run:
    """One workload on this rank's GPU."""

    def __init__(self, wl, weights_dev, torch, moe):
        self.wl, self.torch, self.moe = wl, torch, moe
        Wg, W1, W3, W2 = weights_dev
        self.layer = moe.MoELayer(torch.from_numpy(wl.Wg).cuda() if Wg is None else Wg, W1, W3, W2, k=wl.k,
                                  capacity_factor=wl.capacity_factor, drop_policy=wl.drop_policy)
        self.x = to_dev_bf16(wl.x, torch)
        self.y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
        self.counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")

    def step(self):
        self.layer.forward(self.x, self.y)

    def kept_and_touched(self):
        self.layer.forward(self.x, self.y, counts=self.counts)
        c = self.counts.cpu().numpy()
        cap = self.wl.capacity
        kept = np.minimum(c, cap) if cap is not None else c
        return int(kept.sum()), int((kept > 0).sum())

    def profiled(self, steps):
        """Average duration (ms) of each stage over `steps` instrumented forwards."""
        torch, moe = self.torch, self.moe
        sums = np.zeros(5)
        sh = self.layer.shape(self.wl.T)
        ws = self.layer.workspace(self.wl.T)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
        torch.cuda.synchronize()
        for i in range(steps):
            st = moe.moe_layer_forward_profiled(sh, self.x, self.layer.Wg, self.layer.W1, self.layer.W3,
                                                self.layer.W2, self.y, evs[i], ws, ws.numel())
            moe.check(st, "moe_layer_forward_profiled")
        torch.cuda.synchronize()
        self.clock_mhz = gemm_clocks(ws)
        for i in range(steps):
            sums += [evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(5)]
        return dict(zip(["router", "capacity_and_permute", "gemm1_swiglu", "gemm2", "combine"],
                        (sums / steps).tolist()))

    def twin(self):
        """A second layer on the same weights with its own workspace."""
        wl, L = self.wl, self.layer
        return self.moe.MoELayer(L.Wg, L.W1, L.W3, L.W2, k=wl.k, capacity_factor=wl.capacity_factor,
                                 drop_policy=wl.drop_policy)

    def e2e(self, steps, dist):
        """Tokens/s through the host-buffer entry point (moe_layer_forward_host
        here) with page-locked host x and y, one call after another on one
        stream: every step copies its x in, runs the layer and copies its y out
        before the next step starts (from 4096 dropless tokens the call itself
        overlaps its groups' copies with the other groups' kernels, on the
        library's copy streams; its work ends on this stream)."""
        torch, moe = self.torch, self.moe
        wl, L = self.wl, self.layer
        s_ = torch.cuda.Stream()
        xh = torch.from_numpy(np.ascontiguousarray(wl.x).view(np.int16)).view(torch.bfloat16).pin_memory()
        yh = torch.empty(wl.T, wl.d, dtype=torch.bfloat16).pin_memory()
        for _ in range(2):
            L.forward_host(xh, yh, s_)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(s_)
        for _ in range(steps):
            L.forward_host(xh, yh, s_)
        end.record(s_)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        ms = max_over_ranks(start.elapsed_time(end), torch, dist)
        if L.device_status(wl.T) != moe.MOE_OK:
            raise RuntimeError("device status after the end-to-end run")
        nbytes = wl.T * wl.d * 2
        return ms, nbytes, nbytes

    def e2e_pipelined(self, steps, dist):
        """As e2e, but consecutive steps alternate between two streams (each
        with its own workspace and host buffers), so one step's copies overlap
        another step's kernels: a throughput, not a per-call time."""
        torch, moe = self.torch, self.moe
        wl = self.wl
        L = self.layer
        layers = [L, self.twin()]
        streams = [torch.cuda.Stream(), torch.cuda.Stream()]
        xh = [torch.from_numpy(np.ascontiguousarray(wl.x).view(np.int16)).view(torch.bfloat16).pin_memory()
              for _ in range(2)]
        yh = [torch.empty(wl.T, wl.d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        for i in range(2):
            layers[i].forward_host(xh[i], yh[i], streams[i])
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        cur = torch.cuda.current_stream()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(cur)
        for s_ in streams:
            s_.wait_event(start)
        for i in range(steps):
            j = i & 1
            layers[j].forward_host(xh[j], yh[j], streams[j])
        for s_ in streams:
            ev = torch.cuda.Event()
            ev.record(s_)
            cur.wait_event(ev)
        end.record(cur)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        ms = max_over_ranks(start.elapsed_time(end), torch, dist)
        for i in range(2):
            if layers[i].device_status(wl.T) != moe.MOE_OK:
                raise RuntimeError("device status after the end-to-end run")
        nbytes = wl.T * wl.d * 2
        return ms, nbytes, nbytes


class RunQ4(Run):
    """The decode workload with 4-bit expert weights (quantised on the device
    by moe_quantize_q4 from the same bf16 weights)."""

    def __init__(self, wl, weights_dev, torch, moe):
        self.wl, self.torch, self.moe = wl, torch, moe
        _, W1, W3, W2 = weights_dev
        self.layer = moe.MoELayerQ4.from_bf16(torch.from_numpy(wl.Wg).cuda(), W1, W3, W2, k=wl.k,
                                              capacity_factor=wl.capacity_factor, drop_policy=wl.drop_policy)
        self.x = to_dev_bf16(wl.x, torch)
        self.y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
        self.counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")

    def profiled(self, steps):
        torch, moe = self.torch, self.moe
        L = self.layer
        sums = np.zeros(5)
        sh, ws = L.shape(self.wl.T), L.workspace(self.wl.T)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
        torch.cuda.synchronize()
        for i in range(steps):
            moe.check(moe.moe_layer_forward_q4_profiled(sh, self.x, L.Wg, L.q1, L.q3, L.q2, self.y, evs[i], ws,
                                                        ws.numel()), "moe_layer_forward_q4_profiled")
        torch.cuda.synchronize()
        self.clock_mhz = gemm_clocks(ws)
        for i in range(steps):
            sums += [evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(5)]
        return dict(zip(["router", "capacity_and_permute", "gemm1_swiglu", "gemm2", "combine"],
                        (sums / steps).tolist()))

    def twin(self):
        wl, L = self.wl, self.layer
        return self.moe.MoELayerQ4(L.Wg, L.q1, L.q3, L.q2, k=wl.k, capacity_factor=wl.capacity_factor,
                                   drop_policy=wl.drop_policy)


def gemm_clocks(ws) -> dict:
    """SM clock (MHz) each expert GEMM of the last profiled call ran at: the
    profiled entry points store {clock64, globaltimer ns} of CTA 0 at entry
    and exit of both GEMMs in bytes 64 .. 127 of the workspace."""
    rec = ws[64:128].view(dtype=__import__("torch").int64).cpu().numpy().astype(np.float64)
    out = {}
    for name, (c0, n0, c1, n1) in (("gemm1", rec[0:4]), ("gemm2", rec[4:8])):
        out[name] = (c1 - c0) / (n1 - n0) * 1e3 if n1 > n0 else None
    return out


def clock_peak_tflops(mhz, sms=148, flop_per_clk_sm=8192):
    """Dense bf16 tensor peak at a given SM clock (TFLOP/s)."""
    return sms * flop_per_clk_sm * mhz * 1e-6 if mhz else None


def expert_bytes(d, f):
    return 3 * d * f * 2


def expert_bytes_q4(d, f):
    """codes (half a byte per weight) + one bf16 scale per 64 weights"""
    return 3 * (d * f // 2 + (d * f // 64) * 2)


def cpu_baseline(wl, n_sample=None):
    """The oracle on the host cores: routing of every token plus the expert
    FFN of a seeded sample of tokens (two per oracle thread unless given, so
    that no thread idles); tokens/s scaled to the whole batch."""
    import oracle
    o = oracle.Oracle()
    n_sample = n_sample or 2 * o.num_threads()
    t0 = time.perf_counter()
    r = o.route(wl.x, wl.Wg, wl.k, wl.capacity_factor, wl.drop_policy)
    t_route = time.perf_counter() - t0
    rows = np.random.default_rng(123).choice(wl.T, size=min(n_sample, wl.T), replace=False)
    t0 = time.perf_counter()
    o.layer_rows(wl.x, wl.W1, wl.W3, wl.W2, r, rows)
    t_ffn = time.perf_counter() - t0
    n = len(rows)
    per_token = t_ffn / n + t_route / wl.T
    return dict(value=1.0 / per_token, unit="tokens/s", cores=o.num_threads(), kind="oracle",
                sample=f"routing of all {wl.T} tokens ({t_route:.2f} s) + expert FFN of {n} seeded tokens "
                       f"({t_ffn:.2f} s), fp64, {wl.name}; tokens/s = 1 / (t_ffn/{n} + t_route/{wl.T})")


def make_workload(name, rank, T=None):
    wl = synth.workload(name, T=T)
    wl.seed = 0
    wl.generate(weights=False)
    if rank:
        # every rank routes its own tokens (same weights)
        wl.x = synth.normal_bf16(1000 + rank, synth.TID_X, (wl.T, wl.d))
    return wl


def workload_desc(wl):
    cap = "dropless" if wl.capacity_factor <= 0 else f"capacity factor {wl.capacity_factor}"
    return f"{wl.name}: T={wl.T} d_model={wl.d} d_ff={wl.f} E={wl.E} top-{wl.k} {cap}"


def bench_config(wl, world: int) -> dict:
    """The `config` of both arms' lines (identical for the same workload and N)."""
    return dict(workload=workload_desc(wl), T=wl.T, d_model=wl.d, d_ff=wl.f, E=wl.E, k=wl.k,
                parallelism=f"dp{world} (token shards, weights replicated)" if world > 1 else "single GPU",
                l2="inputs larger than L2: 2.82 GB of expert weights streamed every step; "
                   "ms_per_step_median_l2_flushed: median of per-step events with L2 flushed before each step")


# ---------------------------------------------------------------- arms

def run_reference(args):
    """The CPU oracle as it stands, on rank 0; other ranks exit 0."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    if "WORLD_SIZE" in os.environ and os.environ.get("OMP_NUM_THREADS") == "1":
        # torchrun's one-thread default: the other ranks exit at once, so
        # rank 0 may use every host core
        os.environ["OMP_NUM_THREADS"] = str(os.cpu_count() or 1)
    wl = synth.workload("prefill")
    wl.generate(weights=True)
    import oracle
    o = oracle.Oracle()
    n_sample = 2 * o.num_threads()
    rng = np.random.default_rng(7)

    def one_step():
        """(seconds of the step, seconds per token) of the oracle on this
        step's sample: routing of every token + the FFN of n_sample tokens."""
        t0 = time.perf_counter()
        r = o.route(wl.x, wl.Wg, wl.k, wl.capacity_factor, wl.drop_policy)
        t_route = time.perf_counter() - t0
        rows = rng.choice(wl.T, size=n_sample, replace=False)
        t0 = time.perf_counter()
        o.layer_rows(wl.x, wl.W1, wl.W3, wl.W2, r, rows)
        t_ffn = time.perf_counter() - t0
        return t_route + t_ffn, t_ffn / n_sample + t_route / wl.T

    for _ in range(args.warmup):
        one_step()
    res = [one_step() for _ in range(args.steps)]
    step_s = float(np.mean([a for a, _ in res]))
    per_token = float(np.mean([b for _, b in res]))
    value = 1.0 / per_token
    sample = (f"per step: routing of all {wl.T} tokens + expert FFN of {n_sample} seeded tokens "
              f"(2 per oracle thread), fp64 oracle; tokens/s = 1 / (t_ffn/{n_sample} + t_route/{wl.T})")
    line = dict(metric=METRIC, value=value, unit="tokens/s", n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=step_s * 1e3, higher_is_better=True, scaling="weak",
                vs_baseline=None, dtype="f64", data="synthetic", impl="reference",
                config=bench_config(wl, args.gpus),
                ms_per_step_note=f"measured time of one step's sample ({n_sample} tokens' FFN + routing of all "
                                 f"{wl.T}); the whole batch would take ms_full_batch_estimate",
                ms_full_batch_estimate=per_token * wl.T * 1e3,
                cpu_baseline=dict(value=value, unit="tokens/s", cores=o.num_threads(), kind="oracle",
                                  sample=sample),
                e2e=dict(value=value, unit="tokens/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


def run_dry(args):
    """Launcher and rank plumbing without a GPU: every rank joins a gloo
    group and reports a fixed step time (1 ms + rank); rank 0 prints the max
    over ranks and the whole-job value."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        dist = tdist
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but {world} ranks")
    ms = max_over_ranks(1.0 + rank, torch, dist, device="cpu")
    if dist is not None:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(dict(dry_run=True, n_gpus=world, ranks_seen=world, ms_per_step=ms,
                              value=weak_scaling_value(world, 4096, ms))), flush=True)


def stage_report(wl, q, world, peaks, kernel, traffic_kernel, workload_key, q4=False):
    """The decode-shaped sub-line (HBM roofline of the gate/up GEMM)."""
    d, f, E = wl.d, wl.f, wl.E
    ebytes = expert_bytes_q4(d, f) if q4 else expert_bytes(d, f)
    g1_bytes = q["touched"] * 2 * ebytes // 3 + q["N"] * d * 2 + q["N"] * f * 2
    layer_bytes = q["touched"] * ebytes + wl.T * d * 2 * 2 + E * d * 4 + 2 * q["N"] * f * 2
    g1_ms = q["stages"]["gemm1_swiglu"]
    return dict(workload=workload_desc(wl) + (", 4-bit expert weights (one bf16 scale per 64)" if q4 else ""),
                value=weak_scaling_value(world, wl.T, q["ms"]), unit="tokens/s", ms_per_step=q["ms"],
                ms_per_step_median_l2_flushed=q["ms_flushed"], stage_ms=q["stages"],
                layer_gbs=layer_bytes / (q["ms"] * 1e-3) / 1e9,
                layer_frac_hbm=layer_bytes / (q["ms"] * 1e-3) / 1e9 / peaks["hbm"],
                roofline=dict(bound="hbm", kernel=kernel, achieved=g1_bytes / (g1_ms * 1e-3) / 1e9,
                              peak=peaks["hbm"], unit="GB/s", frac=g1_bytes / (g1_ms * 1e-3) / 1e9 / peaks["hbm"],
                              traffic=traffic_record(traffic_kernel, workload_key),
                              peak_source=f"{peaks['source']} HBM copy bandwidth"),
                e2e=dict(value=weak_scaling_value(world, wl.T, q["e2e_ms"]), unit="tokens/s",
                         h2d_bytes_per_step=q["h2d"], d2h_bytes_per_step=q["d2h"],
                         entry_point=q["entry"]),
                e2e_pipelined=dict(value=weak_scaling_value(world, wl.T, q["e2e_pipe_ms"]), unit="tokens/s",
                                   note="two streams, consecutive steps overlap"),
                experts_touched=q["touched"], gemm_clock_mhz=q["gemm_clock_mhz"])


def run_ours(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but {world} ranks (launch with torchrun or without WORLD_SIZE)")
    dist = None
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    import sparse_mixture_experts_13_b200 as moe
    moe.lib()  # fails loudly if the CUDA library is missing
    peaks = load_peaks()

    # shared seed-0 expert weights
    wl0 = synth.workload("prefill")
    W1 = synth.normal_bf16(0, synth.TID_W1, (8, wl0.f, wl0.d), 0.0, 1.0 / np.sqrt(wl0.d))
    W3 = synth.normal_bf16(0, synth.TID_W3, (8, wl0.f, wl0.d), 0.0, 1.0 / np.sqrt(wl0.d))
    W2 = synth.normal_bf16(0, synth.TID_W2, (8, wl0.d, wl0.f), 0.0, 1.0 / np.sqrt(wl0.f))
    Wd = (None, to_dev_bf16(W1, torch), to_dev_bf16(W3, torch), to_dev_bf16(W2, torch))

    props = torch.cuda.get_device_properties(local)
    pci = None
    if hasattr(props, "pci_bus_id"):
        pci = f"{int(getattr(props, 'pci_domain_id', 0)):08x}:{int(props.pci_bus_id):02x}:" \
              f"{int(getattr(props, 'pci_device_id', 0)):02x}.0"
    sampler = make_clock_sampler(pci)
    sampler.start()
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device="cuda")

    out = {}
    # decode first: the light, bandwidth-bound workload is measured before the
    # power-capped prefill phase heats the GPU; a short pause separates them
    for name in ("decode", "decode_q4", "prefill"):
        time.sleep(1.0)
        wl = make_workload("decode" if name == "decode_q4" else name, rank)
        run = (RunQ4 if name == "decode_q4" else Run)(wl, Wd, torch, moe)
        N, touched = run.kept_and_touched()
        for _ in range(args.warmup):
            run.step()
        with sampler_region(sampler, name):
            ms = time_steps(run.step, args.steps, torch, dist) / args.steps
            stages = run.profiled(args.steps)
            e2e_ms, h2d, d2h = run.e2e(args.steps, dist)
            e2e_pipe_ms, _, _ = run.e2e_pipelined(args.steps, dist)
        ms_flushed = flushed_median_ms(run.step, max(args.steps, 20), torch, flush, dist)
        out[name] = dict(wl=wl, ms=ms, stages=stages, N=N, touched=touched, e2e_ms=e2e_ms / args.steps,
                         gemm_clock_mhz=run.clock_mhz,
                         e2e_pipe_ms=e2e_pipe_ms / args.steps, h2d=h2d, d2h=d2h, ms_flushed=ms_flushed,
                         entry="moe_layer_forward_q4_host" if name == "decode_q4" else "moe_layer_forward_host")
        del run
        torch.cuda.empty_cache()
    clocks = sampler.stop()
    del flush

    line = None
    if rank == 0:
        p = out["prefill"]
        wl = p["wl"]
        d, f, E = wl.d, wl.f, wl.E
        flops_layer = 6.0 * p["N"] * d * f + 2.0 * wl.T * d * E
        g1_flops = 4.0 * p["N"] * d * f
        g1_ms = p["stages"]["gemm1_swiglu"]
        long_run = args.steps * p["ms"] > 1000.0
        peak_tf = peaks["bf16_sustained"] if long_run else peaks["bf16"]
        achieved_tf = g1_flops / (g1_ms * 1e-3) / 1e12
        tr = traffic_record("expert_gemm_pair_kernel<0,2>", "prefill")
        value = weak_scaling_value(world, wl.T, p["ms"])
        tflops = flops_layer / (p["ms"] * 1e-3) / 1e12
        # the SM clock the gate/up GEMM ran at (in-kernel records), else NVML's median
        pre_clk = p["gemm_clock_mhz"].get("gemm1") or (clocks.get("by_region") or {}).get("prefill", {}).get("sm_mhz")
        dec = stage_report(out["decode"]["wl"], out["decode"], world, peaks,
                           "gate/up-projection GEMM (SwiGLU fused)", "expert_gemm_kernel<2,16>", "decode")
        dec_q4 = stage_report(out["decode_q4"]["wl"], out["decode_q4"], world, peaks,
                              "4-bit gate/up-projection GEMM (integer MMA, SwiGLU fused)", "expert_gemm_q4i8_kernel<0,16>",
                              "decode_q4", q4=True)
        # router, grouping, gate/up GEMM, down GEMM, combine; the grouping's
        # row copy runs as its own kernel above 1024 slots; capacity by
        # probability adds its select kernel
        kernels_per_step = (5 + (1 if wl.T * wl.k > 1024 else 0) +
                            (1 if (wl.capacity_factor > 0 and wl.drop_policy == 0) else 0))
        line = dict(
            metric=METRIC, value=value, unit="tokens/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
            ms_per_step=p["ms"], ms_per_step_median_l2_flushed=p["ms_flushed"], higher_is_better=True,
            scaling="weak", vs_baseline=None, dtype="bf16",
            data="synthetic (seeded counter-based N(0,1) tokens, random-init Mixtral-shaped expert weights)",
            config=bench_config(wl, world),
            tflops=tflops,
            tflops_per_ghz=tflops / (pre_clk / 1000.0) if pre_clk else None,
            frac_layer_of_peak=tflops / peak_tf,
            stage_ms=p["stages"],
            roofline=dict(bound="tensor", kernel="gate/up-projection GEMM (SwiGLU fused)", achieved=achieved_tf,
                          peak=peak_tf, unit="TFLOP/s", frac=achieved_tf / peak_tf, traffic=tr,
                          sm_mhz_in_kernel=p["gemm_clock_mhz"].get("gemm1"),
                          frac_of_peak_at_that_clock=(achieved_tf / clock_peak_tflops(p["gemm_clock_mhz"]["gemm1"])
                                                      if p["gemm_clock_mhz"].get("gemm1") else None),
                          peak_source=f"{peaks['source']} bf16 dense "
                                      f"({'sustained' if long_run else 'burst'})"),
            e2e=dict(value=weak_scaling_value(world, wl.T, p["e2e_ms"]), unit="tokens/s", h2d_bytes_per_step=p["h2d"],
                     d2h_bytes_per_step=p["d2h"], entry_point=p["entry"],
                     note="one call after another on one stream; each call copies x in and y out around the layer (in token groups whose copies overlap the other groups' kernels from 4096 dropless tokens)"),
            e2e_pipelined=dict(value=weak_scaling_value(world, wl.T, p["e2e_pipe_ms"]), unit="tokens/s",
                               note="two streams, consecutive steps overlap"),
            gpu_launches=kernels_per_step * args.steps,
            clocks=clocks,
            decode=dec,
            decode_q4=dec_q4,
        )
        if world == 1 and not args.no_cpu_baseline:
            wl.W1, wl.W3, wl.W2 = W1, W3, W2
            line["cpu_baseline"] = cpu_baseline(wl)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


def run_sweep(args):
    """One JSON line per workload (tiny, decode, prefill, skew, sweep T), on
    one GPU: tokens/s, TFLOP/s, GB/s, roofline fractions, per-stage times,
    the SM clock during the timed loop and a sampled oracle baseline.  Not the
    driver's contract line."""
    import torch
    import sparse_mixture_experts_13_b200 as moe
    moe.lib()
    peaks = load_peaks()
    d, f, E = synth.MIXTRAL_D, synth.MIXTRAL_F, 8
    W1 = synth.normal_bf16(0, synth.TID_W1, (E, f, d), 0.0, 1.0 / np.sqrt(d))
    W3 = synth.normal_bf16(0, synth.TID_W3, (E, f, d), 0.0, 1.0 / np.sqrt(d))
    W2 = synth.normal_bf16(0, synth.TID_W2, (E, d, f), 0.0, 1.0 / np.sqrt(f))
    Wd = (None, to_dev_bf16(W1, torch), to_dev_bf16(W3, torch), to_dev_bf16(W2, torch))
    sampler = make_clock_sampler(None)
    sampler.start()
    cases = [("tiny", None), ("decode", None), ("prefill", None), ("skew", None)] + \
            [("sweep", T) for T in synth.SWEEP_T]
    for name, T in cases:
        # a second of idle between workloads, so that one workload's power-capped
        # clock does not carry into the next
        torch.cuda.synchronize()
        time.sleep(1.0)
        wl = synth.workload(name, T=T)
        wl.generate(weights=(name == "tiny"))
        if name == "tiny":
            wd = (None, to_dev_bf16(wl.W1, torch), to_dev_bf16(wl.W3, torch), to_dev_bf16(wl.W2, torch))
        else:
            wd = Wd
            wl.W1, wl.W3, wl.W2 = W1, W3, W2
        run = Run(wl, wd, torch, moe)
        N, touched = run.kept_and_touched()
        for _ in range(args.warmup):
            run.step()
        tag = f"{name}{'' if T is None else T}"
        with sampler_region(sampler, tag):
            ms = time_steps(run.step, args.steps, torch) / args.steps
        stages = run.profiled(args.steps)
        flops = 6.0 * N * wl.d * wl.f + 2.0 * wl.T * wl.d * wl.E
        g1_mhz = run.clock_mhz.get("gemm1")
        wbytes = touched * 3 * wl.d * wl.f * 2
        bytes_ = wbytes + 2 * wl.T * wl.d * 2 + wl.E * wl.d * 4 + 2 * N * wl.f * 2 + 2 * N * wl.d * 2
        tfs = flops / (ms * 1e-3) / 1e12
        gbs = bytes_ / (ms * 1e-3) / 1e9
        line = dict(workload=workload_desc(wl), T=wl.T, kept_slots=N, experts_touched=touched,
                    ms_per_step=ms, tokens_per_s=wl.T / (ms * 1e-3), tflops=tfs, gbs=gbs,
                    frac_bf16_burst=tfs / peaks["bf16"], frac_hbm=gbs / peaks["hbm"], stage_ms=stages,
                    gemm_clock_mhz=run.clock_mhz, peaks_source=peaks["source"],
                    gemm1_frac_of_peak_at_its_clock=(4.0 * N * wl.d * wl.f / (stages["gemm1_swiglu"] * 1e-3) / 1e12
                                                     / clock_peak_tflops(g1_mhz)) if g1_mhz else None)
        if hasattr(sampler, "samples"):
            rows = [r for r in sampler.samples if r[0] == tag]
            line["clocks"] = sampler._summary(rows)
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, n_sample=min(16, wl.T))
        print(json.dumps(line), flush=True)
        del run
        torch.cuda.empty_cache()
    sampler.stop()


# Peer copy bandwidth per direction measured on this machine's B200s over
# NVLink 5 (nominal 900 GB/s): the reference for the dispatch and return.
NVLINK_PEER_GBS = 770.0


def run_ep(args):
    """Expert-parallel arm: the E experts are split over the ranks (E / world
    each, same seed-0 weights as the other arms), every rank routes its own T
    tokens (prefill shape, seed 1 + rank), stores each row straight into the
    receive buffer of its expert's owner (peer stores into symmetric memory),
    runs its experts and reads the results back from the owners.  One JSON
    line: tokens/s over all ranks, the phase times, and the bytes that cross
    between GPUs per step against the peer-copy bandwidth."""
    import datetime
    import torch
    import torch.distributed as tdist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but {world} ranks")
    torch.cuda.set_device(local)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    if "MASTER_PORT" not in os.environ:
        os.environ["MASTER_PORT"] = str(free_port())
    tdist.init_process_group("nccl", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=300),
                             device_id=torch.device("cuda", local))
    import sparse_mixture_experts_13_b200 as moe
    from sparse_mixture_experts_13_b200.ep import EPLayer
    moe.lib()
    wl0 = synth.workload("prefill")
    E, d, f, k, T = wl0.E, wl0.d, wl0.f, wl0.k, args.ep_tokens
    if E % world:
        raise SystemExit(f"{E} experts do not split over {world} ranks")
    epr = E // world
    lo_e = rank * epr
    W1 = synth.normal_bf16(0, synth.TID_W1, (E, f, d), 0.0, 1.0 / np.sqrt(d))[lo_e:lo_e + epr]
    W3 = synth.normal_bf16(0, synth.TID_W3, (E, f, d), 0.0, 1.0 / np.sqrt(d))[lo_e:lo_e + epr]
    W2 = synth.normal_bf16(0, synth.TID_W2, (E, d, f), 0.0, 1.0 / np.sqrt(f))[lo_e:lo_e + epr]
    Wg = torch.from_numpy(synth.normal_f32(0, synth.TID_WG, (E, d), 0.0, 1.0 / np.sqrt(d))).cuda()
    x = to_dev_bf16(synth.normal_bf16(1 + rank, synth.TID_X, (T, d)), torch)
    layer = EPLayer(Wg, to_dev_bf16(W1, torch), to_dev_bf16(W3, torch), to_dev_bf16(W2, torch), E, k, T)
    for _ in range(args.warmup):
        layer.forward(x)
    ms = time_steps(lambda: layer.forward(x), args.steps, torch, tdist) / args.steps
    # phases of one more step, and the rows that left this rank
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    torch.cuda.synchronize()
    layer.forward(x, events=evs)
    torch.cuda.synchronize()
    names = ["route_and_plan", "dispatch", "expert_gemms", "combine"]
    phases = {n: max_over_ranks(evs[i].elapsed_time(evs[i + 1]), torch, tdist) for i, n in enumerate(names)}
    counts = layer.last_counts_all.view(world, E).cpu().numpy()
    remote_rows = int(sum(counts[rank, e] for e in range(E) if e // epr != rank))
    remote = torch.tensor([remote_rows], dtype=torch.int64, device="cuda")
    tdist.all_reduce(remote, op=tdist.ReduceOp.MAX)
    bytes_out = int(remote.item()) * d * 2  # the busiest rank's rows sent (and read back)
    tdist.barrier()
    if rank == 0:
        def link(phase):
            gbs = bytes_out / (phases[phase] * 1e-3) / 1e9 if phases[phase] > 0 else 0.0
            return dict(bytes_per_rank=bytes_out, gbs=gbs, peak=NVLINK_PEER_GBS, unit="GB/s",
                        frac=gbs / NVLINK_PEER_GBS, peak_source="measured peer copy per direction on this pool")
        line = dict(metric="expert-parallel MoE-layer tokens/s", value=weak_scaling_value(world, T, ms),
                    unit="tokens/s", n_gpus=world, steps=args.steps, warmup=args.warmup, ms_per_step=ms,
                    higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16", data="synthetic",
                    config=dict(workload=f"expert-parallel: T={T} tokens per rank d_model={d} d_ff={f} E={E} "
                                         f"({epr} per rank) top-{k} dropless",
                                parallelism=f"ep{world}",
                                l2="inputs larger than L2: expert weights streamed every step"),
                    phases_ms=phases, dispatch=link("dispatch"), return_=link("combine"))
        line["return"] = line.pop("return_")
        print(json.dumps(line), flush=True)
    del layer
    tdist.destroy_process_group()


def free_port() -> int:
    import socket
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        return s_.getsockname()[1]


def launch_ranks(args) -> int:
    """Relaunch this script under torchrun with --gpus ranks on this node."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", f"--master-port={free_port()}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="one JSON line per workload (tiny, decode, prefill, skew, T sweep) instead of the contract line")
    ap.add_argument("--dry-run", action="store_true",
                    help="check the rank launcher and plumbing on CPU (gloo): no GPU work")
    ap.add_argument("--ep", action="store_true",
                    help="expert-parallel arm: the experts split over the --gpus ranks (one JSON line)")
    ap.add_argument("--ep-tokens", type=int, default=4096, help="tokens per rank of the expert-parallel arm")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(launch_ranks(args))
    if args.dry_run:
        run_dry(args)
    elif args.ep:
        run_ep(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

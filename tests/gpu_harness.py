"""Run the CUDA path through the C ABI and compare it with the CPU oracle.

Comparison rules:
* A token is ambiguous when two of its k+1 largest oracle logits lie within
  1e-3 of each other.  There the GPU's (fp32) choice must lie in the oracle's
  near-tie set and keep its order within 1e-3; the oracle is then re-run with
  the GPU's experts for those tokens (conditional oracle), so everything
  downstream is still compared exactly.
* In capacity mode with drop-by-probability, a slot whose probability lies
  within 1e-5 of its expert's threshold is boundary-ambiguous; the oracle
  takes the GPU's keep/drop decision for it, after checking that the GPU kept
  exactly min(count, cap) slots of that expert.
* Then topk_idx, counts, offsets, perm_slot, slot_pos and x_perm are compared
  bit for bit; gate weights within 1e-6; h, y_perm and y by relative
  Frobenius error <= 5e-3 and per element |d| <= 2e-2 * max|ref|.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_mixture_experts_13_b200 as moe
import synth

AMBIG_LOGIT = 1e-3
AMBIG_PROB = 1e-5
REL_FRO = 5e-3
ELEM = 2e-2
W_TOL = 1e-6


def to_dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_f64(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_to_f32(bits).astype(np.float64)


class Device:
    """A workload's inputs on the GPU."""

    def __init__(self, wl: synth.Workload):
        self.wl = wl
        self.x = to_dev_bf16(wl.x)
        self.Wg = torch.from_numpy(wl.Wg).cuda()
        self.W1 = to_dev_bf16(wl.W1)
        self.W3 = to_dev_bf16(wl.W3)
        self.W2 = to_dev_bf16(wl.W2)

    def shape(self, variant=0, T=None):
        wl = self.wl
        return moe.make_shape(wl.T if T is None else T, wl.d, wl.f, wl.E, wl.k, wl.capacity_factor,
                              wl.drop_policy, variant)


class guarded:
    """With the debug library loaded, arm the workspace guards before the
    calls inside the block and check them (and the device status) after;
    with the release library, nothing."""

    def __init__(self, sh, ws, nws, q4=False):
        self.sh, self.ws, self.nws, self.q4 = sh, ws, nws, q4
        self.on = moe.moe_debug_build() == 1

    def __enter__(self):
        if self.on:
            moe.check(moe.moe_debug_workspace_arm(self.sh, self.ws, self.nws, self.q4), "debug_workspace_arm")
        return self

    def __exit__(self, exc_type, exc, tb):
        if self.on and exc_type is None:
            st = moe.moe_debug_workspace_check(self.sh, self.ws, self.nws, self.q4)
            assert st == moe.MOE_OK, f"workspace guard overwritten: {moe.status_string(st)}"
        return False


def run_stages(dev: Device, variant: int = 0) -> dict:
    """Router -> permute -> grouped SwiGLU -> combine through the stage entry points."""
    wl = dev.wl
    T, d, f, E, k = wl.T, wl.d, wl.f, wl.E, wl.k
    S = T * k
    sh = dev.shape(variant)
    cu = lambda *shape, dt: torch.empty(*shape, dtype=dt, device="cuda")
    out = dict(logits=cu(T, E, dt=torch.float32), idx=cu(S, dt=torch.int32), w=cu(S, dt=torch.float32),
               p=cu(S, dt=torch.float32), counts=cu(E, dt=torch.int32), offsets=cu(E + 1, dt=torch.int32),
               slot_pos=cu(S, dt=torch.int32), perm_slot=cu(S, dt=torch.int32),
               x_perm=cu(S, d, dt=torch.bfloat16), h=cu(S, f, dt=torch.bfloat16),
               y_perm=cu(S, d, dt=torch.bfloat16), y=cu(T, d, dt=torch.bfloat16))
    nws = moe.moe_workspace_size(sh)
    ws = cu(nws, dt=torch.uint8)
    o = out
    with guarded(sh, ws, nws):
        moe.check(moe.moe_router_topk(sh, dev.x, dev.Wg, o["logits"], o["idx"], o["w"], o["p"], o["counts"]),
                  "router")
        moe.check(moe.moe_permute(sh, dev.x, o["idx"], o["p"], o["counts"], o["offsets"], o["slot_pos"],
                                  o["perm_slot"], o["x_perm"], ws, nws), "permute")
        moe.check(moe.moe_grouped_swiglu(sh, o["x_perm"], o["offsets"], dev.W1, dev.W3, dev.W2, o["h"],
                                         o["y_perm"], ws, nws), "grouped_swiglu")
        moe.check(moe.moe_combine(sh, o["y_perm"], o["slot_pos"], o["w"], o["y"]), "combine")
    st = moe.moe_read_device_status(ws)
    assert st == moe.MOE_OK, moe.status_string(st)
    torch.cuda.synchronize()
    return {key: v for key, v in out.items()}


def run_layer(dev: Device, variant: int = 0, reps: int = 1) -> dict:
    wl = dev.wl
    sh = dev.shape(variant)
    nws = moe.moe_workspace_size(sh)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(wl.T * wl.k, dtype=torch.int32, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    ys = []
    for _ in range(reps):
        with guarded(sh, ws, nws):
            moe.check(moe.moe_layer_forward(sh, dev.x, dev.Wg, dev.W1, dev.W3, dev.W2, y, idx, counts, ws, nws),
                      "layer_forward")
        st = moe.moe_read_device_status(ws)
        assert st == moe.MOE_OK, moe.status_string(st)
        ys.append(bf16_host(y).copy())
    return dict(y=ys[0], ys=ys, idx=idx.cpu().numpy(), counts=counts.cpu().numpy())


def near_tie_sets(L: np.ndarray, k: int):
    """Per token: ambiguous flag and the oracle's sorted order."""
    order = np.argsort(-L, axis=1, kind="stable")
    srt = np.take_along_axis(L, order, 1)
    m = min(k + 1, L.shape[1])
    gaps = srt[:, :m - 1] - srt[:, 1:m] if m > 1 else np.full((L.shape[0], 1), np.inf)
    amb = (gaps <= AMBIG_LOGIT).any(axis=1)
    return amb, order, srt


def check_choice_in_tie_set(L_t: np.ndarray, gpu_idx_t: np.ndarray, k: int) -> bool:
    """The GPU's k experts are a valid top-k of L_t up to 1e-3: each chosen
    logit is at least the oracle's k-th largest minus the tolerance, the
    choices are distinct and in non-increasing order up to the tolerance."""
    if len(set(gpu_idx_t.tolist())) != k:
        return False
    srt = np.sort(L_t)[::-1]
    kth = srt[k - 1]
    vals = L_t[gpu_idx_t]
    if (vals < kth - AMBIG_LOGIT).any():
        return False
    return bool((np.diff(vals) <= AMBIG_LOGIT).all())


def conditional_route(o: oracle.Oracle, wl: synth.Workload, gpu_idx: np.ndarray, gpu_p: np.ndarray,
                      gpu_slot_pos: np.ndarray, stats: dict | None = None) -> dict:
    """Oracle routing, taking the GPU's choices on ambiguous tokens / slots."""
    T, k, E = wl.T, wl.k, wl.E
    L = o.router_logits(wl.x, wl.Wg)
    amb, order, _ = near_tie_sets(L, k)
    gi = gpu_idx.reshape(T, k)
    base_idx = order[:, :k].astype(np.int32)
    bad = np.nonzero((~amb) & (gi != base_idx).any(1))[0]
    assert bad.size == 0, f"top-k differs on unambiguous tokens {bad[:10]}: gpu {gi[bad[:3]]} oracle {base_idx[bad[:3]]}"
    override = np.full((T, k), -1, np.int32)
    for t in np.nonzero(amb)[0]:
        assert check_choice_in_tie_set(L[t], gi[t], k), (t, L[t], gi[t])
        override[t] = gi[t]
    r = o.route(wl.x, wl.Wg, k, wl.capacity_factor, wl.drop_policy, idx_override=override, logits=L)
    n_kept_override = 0
    if r["cap"] is not None and wl.drop_policy == oracle.DROP_BY_PROB:
        gpu_kept = (gpu_slot_pos >= 0).astype(np.int64)
        kept_override = np.full(T * k, -1, np.int64)
        idx_f = r["idx"].ravel()
        p_f = r["p"].ravel()
        for e in range(E):
            slots = np.nonzero(idx_f == e)[0]
            if slots.size <= r["cap"]:
                continue
            assert gpu_kept[slots].sum() == r["cap"], (e, gpu_kept[slots].sum(), r["cap"])
            ps = np.sort(p_f[slots])[::-1]
            thr = ps[r["cap"] - 1]
            near = slots[np.abs(p_f[slots] - thr) <= AMBIG_PROB]
            if near.size:
                # the GPU's choice among the near-threshold slots must keep the
                # right number of them
                kept_override[near] = gpu_kept[near]
                n_kept_override += int(near.size)
        if n_kept_override:
            r = o.route(wl.x, wl.Wg, k, wl.capacity_factor, wl.drop_policy, idx_override=override,
                        kept_override=kept_override, logits=L)
    if stats is not None:
        stats.update(ambiguous_tokens=int(amb.sum()), boundary_slots=n_kept_override)
    return r


def rel_fro(a: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / den) if den > 0 else float(np.linalg.norm(a))


def assert_close(a: np.ndarray, ref: np.ndarray, what: str):
    if ref.size == 0:
        return
    rf = rel_fro(a, ref)
    mx = float(np.abs(ref).max())
    err = float(np.abs(a - ref).max())
    assert rf <= REL_FRO, f"{what}: relative Frobenius {rf:.3e} > {REL_FRO}"
    assert err <= ELEM * mx + 1e-30, f"{what}: max |d| {err:.3e} > {ELEM} * {mx:.3e}"


def compare_routing(gpu: dict, r: dict, wl: synth.Workload):
    """Bit-exact comparison of the integer outputs; gates within 1e-6."""
    T, k, E = wl.T, wl.k, wl.E
    g = {key: (v.cpu().numpy() if isinstance(v, torch.Tensor) and key not in ("x_perm", "h", "y_perm", "y")
               else v) for key, v in gpu.items()}
    assert np.array_equal(g["idx"].reshape(T, k), r["idx"]), "topk_idx"
    assert np.array_equal(g["counts"], r["counts"]), ("counts", g["counts"], r["counts"])
    assert np.array_equal(g["offsets"], r["offsets"]), ("offsets", g["offsets"], r["offsets"])
    N = int(r["offsets"][E])
    assert np.array_equal(g["perm_slot"][:N], r["perm_slot"]), "perm_slot"
    assert np.array_equal(g["slot_pos"], r["slot_pos"]), "slot_pos"
    assert np.abs(g["w"].reshape(T, k) - r["w"]).max() <= W_TOL, ("topk_w", np.abs(g["w"].reshape(T, k) - r["w"]).max())
    if "logits" in g:
        assert np.abs(g["logits"] - r["logits"]).max() <= 1e-4
    # x_perm rows are exact copies of the routed tokens' rows
    xp = bf16_host(gpu["x_perm"])[:N]
    assert np.array_equal(xp, wl.x[r["perm_slot"] // k]), "x_perm"
    return N


def sample_tokens(wl: synth.Workload, r: dict, n: int, seed: int = 1, block_rows: int | None = None) -> np.ndarray:
    """n random token indices, plus: dropped tokens when there are any, the
    first and last token, and -- with block_rows, the token-block height of
    the GEMM schedule in use -- the token of one random row in every
    (expert, token block) tile and of the last row of every expert, so that
    every tile of both GEMMs (a full row of h or y_perm spans all weight
    blocks) and every partial last block is checked."""
    T, k = wl.T, wl.k
    if T <= n:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(T, size=n, replace=False).tolist())
    dropped = np.nonzero((r["slot_pos"].reshape(T, k) < 0).any(1))[0]
    for t in dropped[: max(1, n // 4)]:
        pick.add(int(t))
    pick.update({0, T - 1})
    if block_rows:
        off, perm = r["offsets"], r["perm_slot"]
        for e in range(len(off) - 1):
            lo, hi = int(off[e]), int(off[e + 1])
            for b0 in range(lo, hi, block_rows):
                row = int(rng.integers(b0, min(hi, b0 + block_rows)))
                pick.add(int(perm[row]) // k)
            if hi > lo:
                pick.add(int(perm[hi - 1]) // k)
    return np.array(sorted(pick), np.int64)


def schedule_block_rows(T: int, variant: int, k: int = 2, E: int = 8) -> int:
    """Token rows per tile of the expert GEMMs, as the library chooses them:
    the streaming schedule's token tile (twice the mean slots per expert,
    rounded up to 16; AUTO takes it for T <= 128), 128 for single-CTA tiles
    (AUTO while T k / E <= 112), 256 for CTA pairs."""
    if variant == 0:
        variant = 2 if T <= 128 else 3 if T * k <= 112 * E else 1
    if variant == 2:
        b = max(16, ((2 * ((T * k + E - 1) // E) + 15) // 16) * 16)
        return 16 if b <= 16 else 32 if b <= 32 else 64 if b <= 64 else 128
    return 128 if variant == 3 else 256


# ------------------------------------------------------------ 4-bit experts

class QDevice(Device):
    """A workload's inputs on the GPU with the expert weights in the 4-bit
    format, quantised by the oracle (the GPU consumes the oracle's bytes)."""

    def __init__(self, wl: synth.Workload, o: oracle.Oracle, q=None):
        self.wl = wl
        self.x = to_dev_bf16(wl.x)
        self.Wg = torch.from_numpy(wl.Wg).cuda()
        self.q_host = q if q is not None else tuple(o.q4_quantize(W) for W in (wl.W1, wl.W3, wl.W2))
        self.q = tuple((torch.from_numpy(c).cuda(), to_dev_bf16(s)) for c, s in self.q_host)


def run_layer_q4(dev: QDevice, reps: int = 1) -> dict:
    wl = dev.wl
    sh = dev.shape(0)
    nws = moe.moe_workspace_size_q4(sh)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(wl.T * wl.k, dtype=torch.int32, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    ys = []
    for _ in range(reps):
        with guarded(sh, ws, nws, q4=True):
            moe.check(moe.moe_layer_forward_q4(sh, dev.x, dev.Wg, *dev.q, y, idx, counts, ws, nws),
                      "layer_forward_q4")
        st = moe.moe_read_device_status(ws)
        assert st == moe.MOE_OK, moe.status_string(st)
        ys.append(bf16_host(y).copy())
    return dict(y=ys[0], ys=ys, idx=idx.cpu().numpy(), counts=counts.cpu().numpy())


def run_stages_q4(dev: QDevice) -> dict:
    """Router -> permute -> 4-bit grouped SwiGLU -> combine through the stage entry points."""
    wl = dev.wl
    T, d, f, E, k = wl.T, wl.d, wl.f, wl.E, wl.k
    S = T * k
    sh = dev.shape(0)
    cu = lambda *shape, dt: torch.empty(*shape, dtype=dt, device="cuda")
    o = dict(idx=cu(S, dt=torch.int32), w=cu(S, dt=torch.float32), p=cu(S, dt=torch.float32),
             counts=cu(E, dt=torch.int32), offsets=cu(E + 1, dt=torch.int32), slot_pos=cu(S, dt=torch.int32),
             perm_slot=cu(S, dt=torch.int32), x_perm=cu(S, d, dt=torch.bfloat16), h=cu(S, f, dt=torch.bfloat16),
             y_perm=cu(S, d, dt=torch.bfloat16), y=cu(T, d, dt=torch.bfloat16))
    nws = max(moe.moe_workspace_size_q4(sh), moe.moe_workspace_size(sh))
    ws = cu(nws, dt=torch.uint8)
    moe.check(moe.moe_router_topk(sh, dev.x, dev.Wg, None, o["idx"], o["w"], o["p"], o["counts"]), "router")
    moe.check(moe.moe_permute(sh, dev.x, o["idx"], o["p"], o["counts"], o["offsets"], o["slot_pos"],
                              o["perm_slot"], o["x_perm"], ws, nws), "permute")
    moe.check(moe.moe_grouped_swiglu_q4(sh, o["x_perm"], o["offsets"], *dev.q, o["h"], o["y_perm"], ws, nws),
              "grouped_swiglu_q4")
    moe.check(moe.moe_combine(sh, o["y_perm"], o["slot_pos"], o["w"], o["y"]), "combine")
    st = moe.moe_read_device_status(ws)
    assert st == moe.MOE_OK, moe.status_string(st)
    torch.cuda.synchronize()
    return o


# ------------------------------------------------- next-best-expert fallback

def gpu_logits(dev: Device) -> np.ndarray:
    """The router's fp32 logits (moe_router_topk with its logits output)."""
    wl = dev.wl
    sh = dev.shape(0)
    S, E = wl.T * wl.k, wl.E
    cu = lambda *shape, dt: torch.empty(*shape, dtype=dt, device="cuda")
    lg = cu(wl.T, E, dt=torch.float32)
    moe.check(moe.moe_router_topk(moe.make_shape(wl.T, wl.d, wl.f, E, wl.k), dev.x, dev.Wg, lg, cu(S, dt=torch.int32),
                                  cu(S, dt=torch.float32), cu(S, dt=torch.float32), cu(E, dt=torch.int32)), "router")
    torch.cuda.synchronize()
    return lg.cpu().numpy().astype(np.float64)


def fallback_route(o: oracle.Oracle, wl: synth.Workload, gpu_idx: np.ndarray, gl: np.ndarray,
                   stats: dict | None = None) -> dict:
    """Oracle routing with the fallback.  A token whose oracle logits have two
    of the 2k+1 largest within 1e-3 is ambiguous: the GPU's router order
    (from its fp32 logits, ties to the smaller index) must order the
    oracle's values within 1e-3, and the oracle then takes that order for the
    token (its top-k and the ranks the fallback reads)."""
    T, k, E = wl.T, wl.k, wl.E
    L = o.router_logits(wl.x, wl.Wg)
    m = min(2 * k + 1, E)
    order = np.argsort(-L, axis=1, kind="stable")
    srt = np.take_along_axis(L, order, 1)
    amb = (srt[:, :m - 1] - srt[:, 1:m] <= AMBIG_LOGIT).any(axis=1) if m > 1 else np.zeros(T, bool)
    gorder = np.argsort(-gl, axis=1, kind="stable")
    gi = gpu_idx.reshape(T, k)
    bad = np.nonzero((~amb) & (gorder[:, :m] != order[:, :m]).any(1))[0]
    assert bad.size == 0, f"router order differs on unambiguous tokens {bad[:10]}"
    assert np.array_equal(gi, gorder[:, :k]), "GPU top-k is not the order of its own logits"
    idx_ov = np.full((T, k), -1, np.int32)
    ord_ov = np.full((T, E), -1, np.int32)
    for t in np.nonzero(amb)[0]:
        vals = L[t, gorder[t, :m]]
        assert (vals >= srt[t, :m] - AMBIG_LOGIT).all() and (np.diff(vals) <= AMBIG_LOGIT).all(), (t, L[t], gorder[t])
        idx_ov[t] = gorder[t, :k]
        ord_ov[t] = gorder[t]
    if stats is not None:
        stats.update(ambiguous_tokens=int(amb.sum()))
    return o.route(wl.x, wl.Wg, k, wl.capacity_factor, wl.drop_policy, idx_override=idx_ov, logits=L,
                   order_override=ord_ov)

"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each pin is a function ``pin_*(o: Oracle)`` that raises AssertionError when
the oracle ``o`` disagrees with the pages' printed values, a closed form, an
invariant, a special case or a brute-force restatement on tiny inputs.  They
run against the real oracle (tests/test_oracle_pins.py) and against builds of
it with a planted mistake, each of which at least one pin must catch.
"""
from __future__ import annotations

import math
import os

import numpy as np

import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name: str) -> dict:
    out: dict = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            out.setdefault(key.strip(), []).append(val.split())
    return {k: (v[0] if len(v) == 1 else v) for k, v in out.items()}


def _bf16(a) -> np.ndarray:
    return synth.f32_to_bf16(np.asarray(a, np.float32))


def _w(bits) -> np.ndarray:
    return synth.bf16_to_f32(bits).astype(np.float64)


def tiny_problem(T=24, d=32, f=48, E=8, seed=7, scale_x=1.0):
    rng = np.random.default_rng(seed)
    x = _bf16(rng.standard_normal((T, d)) * scale_x)
    Wg = rng.standard_normal((E, d)).astype(np.float32) / np.float32(np.sqrt(d))
    W1 = _bf16(rng.standard_normal((E, f, d)) / np.sqrt(d))
    W3 = _bf16(rng.standard_normal((E, f, d)) / np.sqrt(d))
    W2 = _bf16(rng.standard_normal((E, d, f)) / np.sqrt(f))
    return x, Wg, W1, W3, W2


def _np_expert(xr, W1e, W3e, W2e):
    a = _w(W1e) @ xr
    b = _w(W3e) @ xr
    h = a * (1.0 / (1.0 + np.exp(-a))) * b
    return h, _w(W2e) @ h


# ---------------------------------------------------------------- gate pins

def pin_worked_example(o):
    """The worked routing example: experts 0 and 2 (the page's "1 and 3"),
    weights printed as 0.6682 / 0.3318; their exact values are the logistic
    function of the score gap 2.1 - 1.4 = 0.7."""
    g = read_golden("worked_routing_example.txt")
    scores = np.array([[float(v) for v in g["scores"]]])
    k = int(g["k"][0])
    idx = o.topk(scores, k)
    assert idx[0].tolist() == [int(v) for v in g["experts_0based"]], idx
    w, p = o.gates(scores, idx)
    printed = [float(v) for v in g["weights_4dp"]]
    assert [round(float(v), 4) for v in w[0]] == printed, w
    sig = 1.0 / (1.0 + math.exp(-0.7))
    assert abs(w[0, 0] - sig) < 1e-15 and abs(w[0, 1] - (1.0 - sig)) < 1e-15, w
    assert p[0, 0] > p[0, 1] > 0 and p[0].sum() < 1.0


def pin_gate_forms_agree(o):
    """The three gate statements on the pages -- softmax over all E then
    top-k and renormalise; top-k with the rest masked to -inf then softmax;
    softmax over the k kept logits -- are one function.  The first two are
    written here independently and compared with the oracle's gates, which
    also give the full-softmax probability p of each chosen expert."""
    rng = np.random.default_rng(11)
    for E, k in ((8, 2), (8, 1), (16, 4), (4, 4), (32, 3)):
        L = rng.standard_normal((500, E)) * 2.0
        idx = o.topk(L, k)
        w, p = o.gates(L, idx)
        order = np.argsort(-L, axis=1, kind="stable")[:, :k]
        assert np.array_equal(idx, order), (E, k)
        full = np.exp(L - L.max(1, keepdims=True))
        full /= full.sum(1, keepdims=True)
        pk = np.take_along_axis(full, order, 1)
        formA = pk / pk.sum(1, keepdims=True)
        masked = np.full_like(L, -np.inf)
        np.put_along_axis(masked, order, np.take_along_axis(L, order, 1), 1)
        eB = np.exp(masked - masked.max(1, keepdims=True))
        formB = np.take_along_axis(eB / eB.sum(1, keepdims=True), order, 1)
        assert np.allclose(w, formA, rtol=0, atol=1e-14), (E, k)
        assert np.allclose(w, formB, rtol=0, atol=1e-14), (E, k)
        assert np.allclose(p, pk, rtol=0, atol=1e-14), (E, k)
        assert np.allclose(w.sum(1), 1.0, rtol=0, atol=1e-14)


def pin_topk_ties_and_distinct(o):
    """Equal logits go to the smaller expert index; every token gets k
    distinct experts; slot 0 holds the largest logit."""
    L = np.array([[1.0, 3.0, 3.0, 0.5, 3.0, 0.0, 0.0, 0.0],
                  [0.0] * 8,
                  [-1.0, -1.0, -2.0, -1.0, -5.0, -1.0, -1.0, -1.0]])
    idx = o.topk(L, 2)
    assert idx.tolist() == [[1, 2], [0, 1], [0, 1]], idx
    idx3 = o.topk(L, 3)
    assert idx3.tolist() == [[1, 2, 4], [0, 1, 2], [0, 1, 3]], idx3
    rng = np.random.default_rng(3)
    L = rng.standard_normal((300, 8))
    idx = o.topk(L, 2)
    assert np.all(idx[:, 0] != idx[:, 1])
    assert np.all(np.take_along_axis(L, idx[:, :1], 1)[:, 0] >= np.take_along_axis(L, idx[:, 1:], 1)[:, 0])
    w, _ = o.gates(L, o.topk(L, 1))
    assert np.all(w == 1.0)


def pin_router_logits(o):
    """Router logits are the plain product x . Wg^T of the widened inputs
    (compared with numpy's matmul, a different summation order)."""
    x, Wg, *_ = tiny_problem(T=40, d=96)
    L = o.router_logits(x, Wg)
    ref = _w(x) @ Wg.astype(np.float64).T
    assert np.allclose(L, ref, rtol=0, atol=1e-12)
    # one hand-computed case: a basis vector picks a column of Wg
    xb = np.zeros((1, 96), np.uint16)
    xb[0, 5] = 0x3F80
    assert np.array_equal(o.router_logits(xb, Wg)[0], Wg[:, 5].astype(np.float64))


# ------------------------------------------------------ capacity / grouping

def pin_capacity_arithmetic(o):
    """cap = floor(cf*T*k/E): 2560 at T=8192, cf=1.25; at T=1 the page's
    1.25*1/8 = 0.16 slots rounds down to zero, so everything drops."""
    g = read_golden("capacity_example.txt")
    cf, E, k = float(g["cf"][0]), int(g["E"][0]), int(g["k"][0])
    assert round(cf * 1 / E, 2) == float(g["batch1_fraction"][0])
    for T, cap_expect in ([int(a), int(b)] for a, b in g["T_cap"]):
        idx = np.tile(np.arange(k, dtype=np.int32), (T, 1))
        p = np.full((T, k), 0.5)
        kept, cap = o.capacity(idx, p, E, cf, 0)
        assert cap == cap_expect, (T, cap)
        assert kept.sum() == min(T, cap_expect) * k


def _brute_capacity(idx, p, E, cap, policy):
    T, k = idx.shape
    kept = np.zeros(T * k, np.uint8)
    for e in range(E):
        slots = [s for s in range(T * k) if idx.flat[s] == e]
        if policy == 0:
            slots.sort(key=lambda s: (-p.flat[s], s // k))
        for s in slots[:cap]:
            kept[s] = 1
    return kept


def pin_capacity_bruteforce(o):
    """Both drop policies against a brute-force sort, including exact
    probability ties (broken by the smaller token), cf huge (= dropless)
    and cap = 0 (all dropped)."""
    rng = np.random.default_rng(5)
    for trial in range(6):
        T, E, k = 200, 8, 2
        L = rng.standard_normal((T, E))
        L[:, 0] += 1.5 * (trial % 2)                     # skew half of the trials
        idx = o.topk(L, k)
        _, p = o.gates(L, idx)
        if trial >= 4:
            p = np.round(p, 1)                           # many exact ties
        for cf in (0.5, 1.0, 1.25):
            cap = int(np.floor(cf * T * k / E))
            for policy in (0, 1):
                kept, c = o.capacity(idx, p, E, cf, policy)
                assert c == cap
                assert np.array_equal(kept, _brute_capacity(idx, p, E, cap, policy)), (trial, cf, policy)
        kept, c = o.capacity(idx, p, E, 1e9, 0)
        assert kept.all()
        kept, c = o.capacity(idx, p, E, 0.0, 0)
        assert c is None and kept.all()
        kept, c = o.capacity(idx, p, E, 1e-6, 1)
        assert c == 0 and not kept.any()


def pin_grouping_invariants(o):
    """Histogram sums to T*k (the page's 1000 tokens x 2 = 2000 assignments,
    250 per expert when balanced); kept_e = min(count_e, cap); offsets are the
    prefix sums; perm_slot and slot_pos are inverse; rows of one expert are in
    ascending token order."""
    g = read_golden("load_example.txt")
    T, k, E = int(g["tokens"][0]), int(g["k"][0]), int(g["experts"][0])
    balanced = np.array([[(2 * t) % E, (2 * t + 1) % E] for t in range(T)], np.int32)
    perm = o.permute(balanced, np.ones(T * k, np.uint8), E)
    assert perm["counts"].sum() == int(g["assignments"][0])
    assert np.all(perm["counts"] == int(g["balanced_per_expert"][0]))
    assert float(g["skewed_busiest"][0]) / (T * k / E) == float(g["skewed_ratio"][0])
    rng = np.random.default_rng(9)
    for cf in (0.0, 1.0):
        L = rng.standard_normal((T, E))
        L[:, 3] += 1.0
        idx = o.topk(L, k)
        _, p = o.gates(L, idx)
        kept, cap = o.capacity(idx, p, E, cf, 0)
        pm = o.permute(idx, kept, E)
        cnt = np.bincount(idx.ravel(), minlength=E)
        assert np.array_equal(pm["counts"], cnt)
        lim = cnt if cap is None else np.minimum(cnt, cap)
        assert np.array_equal(pm["kept_counts"], lim)
        assert np.array_equal(pm["offsets"], np.concatenate([[0], np.cumsum(lim)]))
        ps, sp = pm["perm_slot"], pm["slot_pos"]
        assert np.array_equal(sp[ps], np.arange(len(ps)))
        assert np.all((sp >= 0) == (kept == 1))
        for e in range(E):
            rows = ps[pm["offsets"][e]:pm["offsets"][e + 1]]
            assert np.all(idx.ravel()[rows] == e)
            assert np.all(np.diff(rows // k) > 0)


# ------------------------------------------------------------- expert pins

def pin_silu_values(o):
    """SiLU(a) = a * sigmoid(a) = a / (1 + e^-a), through a 1x1 expert with
    unit weights (so a = b = x and h = silu(x) * x), and with W3 = 2."""
    one = np.array([0x3F80], np.uint16)
    for xv in (1.0, -2.0, 0.0, 3.5):
        xb = _bf16([xv])
        h, out = o.expert_row(xb, one.reshape(1, 1), one.reshape(1, 1), one.reshape(1, 1))
        # a = b = x, so h = silu(x) * x
        silu = xv / (1.0 + math.exp(-xv))
        assert abs(h[0] - silu * xv) < 1e-15, (xv, h)
        assert out[0] == h[0]
    h, _ = o.expert_row(_bf16([1.0]), one.reshape(1, 1), _bf16([[2.0]]), one.reshape(1, 1))
    assert abs(h[0] - 2.0 / (1.0 + math.exp(-1.0))) < 1e-15


def pin_expert_matmul(o):
    """One expert on one row equals numpy's W2 (silu(W1 x) * W3 x)."""
    x, Wg, W1, W3, W2 = tiny_problem(T=3, d=40, f=56)
    for t in range(3):
        h, out = o.expert_row(x[t], W1[2], W3[2], W2[2])
        hr, orf = _np_expert(_w(x[t]), W1[2], W3[2], W2[2])
        assert np.allclose(h, hr, rtol=1e-12, atol=1e-13)
        assert np.allclose(out, orf, rtol=1e-12, atol=1e-13)


# -------------------------------------------------------------- layer pins

def pin_dense_bruteforce(o):
    """Layer output against the dense statement y = sum_e G(x)_e Expert_e(x)
    with G = softmax over the top-k logits and exactly zero elsewhere, every
    expert evaluated on every token (numpy, independent of the oracle's
    sparse dispatch), and against a restatement of the per-expert mask loop
    (gather the tokens that chose e, run e, add w * out)."""
    for E, k in ((8, 2), (4, 1), (8, 3)):
        x, Wg, W1, W3, W2 = tiny_problem(T=20, d=32, f=48, E=E, seed=E + k)
        r = o.layer(x, Wg, W1, W3, W2, k)
        L = _w(x) @ Wg.astype(np.float64).T
        T = x.shape[0]
        y_dense = np.zeros((T, x.shape[1]))
        for t in range(T):
            top = np.argsort(-L[t], kind="stable")[:k]
            g = np.zeros(E)
            g[top] = np.exp(L[t, top] - L[t, top].max())
            g /= g.sum()
            for e in range(E):
                _, out = _np_expert(_w(x[t]), W1[e], W3[e], W2[e])
                y_dense[t] += g[e] * out
        assert np.allclose(r["y"], y_dense, rtol=1e-12, atol=1e-12), (E, k)
        # mask loop
        y_mask = np.zeros_like(y_dense)
        idx, w = r["idx"], r["w"]
        for e in range(E):
            mask = (idx == e).any(1)
            for t in np.nonzero(mask)[0]:
                pos = int(np.argmax(idx[t] == e))
                _, out = _np_expert(_w(x[t]), W1[e], W3[e], W2[e])
                y_mask[t] += w[t, pos] * out
        assert np.allclose(r["y"], y_mask, rtol=1e-12, atol=1e-12), (E, k)


def pin_special_cases(o):
    """Identical experts give y = Expert(x) whatever the routing (gates sum to
    one); W2 = 0 gives y = 0; doubling W2 (exact in bf16) doubles y exactly;
    with k = E the layer is the dense softmax mixture over all experts."""
    x, Wg, W1, W3, W2 = tiny_problem(T=12, d=32, f=40, E=8, seed=21)
    same = lambda a: np.repeat(a[:1], a.shape[0], 0)
    r = o.layer(x, Wg, same(W1), same(W3), same(W2), 2)
    for t in range(12):
        _, out = _np_expert(_w(x[t]), W1[0], W3[0], W2[0])
        assert np.allclose(r["y"][t], out, rtol=1e-12, atol=1e-13)
    r0 = o.layer(x, Wg, W1, W3, np.zeros_like(W2), 2)
    assert np.all(r0["y"] == 0.0)
    r1 = o.layer(x, Wg, W1, W3, W2, 2)
    r2 = o.layer(x, Wg, W1, W3, _bf16(_w(W2) * 2.0), 2)
    assert np.array_equal(r2["y"], 2.0 * r1["y"])
    rk = o.layer(x, Wg, W1, W3, W2, 8)
    L = _w(x) @ Wg.astype(np.float64).T
    P = np.exp(L - L.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    for t in range(12):
        ref = sum(P[t, e] * _np_expert(_w(x[t]), W1[e], W3[e], W2[e])[1] for e in range(8))
        assert np.allclose(rk["y"][t], ref, rtol=1e-12, atol=1e-13)


def pin_dropped_slots(o):
    """A dropped slot adds nothing and the other gate is not renormalised:
    y(t) = sum over kept slots of w_j * Expert_j(x_t); a token with both slots
    dropped gives y = 0 (it passes through on the residual)."""
    x, Wg, W1, W3, W2 = tiny_problem(T=40, d=32, f=40, E=8, seed=4)
    r = o.route(x, Wg, 2, cf=0.5, policy=0)
    assert r["cap"] == 5
    assert (r["kept"] == 0).any()
    y = o.layer_rows(x, W1, W3, W2, r, np.arange(40))["y"]
    for t in range(40):
        ref = np.zeros(32)
        for j in range(2):
            s = 2 * t + j
            if r["kept"][s]:
                e = r["idx"][t, j]
                ref += r["w"][t, j] * _np_expert(_w(x[t]), W1[e], W3[e], W2[e])[1]
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-13)
        if not r["kept"][2 * t] and not r["kept"][2 * t + 1]:
            assert np.all(y[t] == 0.0)


ALL_PINS = [pin_worked_example, pin_gate_forms_agree, pin_topk_ties_and_distinct,
            pin_router_logits, pin_capacity_arithmetic, pin_capacity_bruteforce,
            pin_grouping_invariants, pin_silu_values, pin_expert_matmul,
            pin_dense_bruteforce, pin_special_cases, pin_dropped_slots]


# ------------------------------------------------------- 4-bit expert weights

def _exact_q4_matrix(rng, E, R, K):
    """Random W [E, R, K] whose every 64-input block is (v * 2^j) with integer
    v in [-7, 7], one |v| = 7 per block and a random exponent j per block:
    exactly representable in the 4-bit format, so quantisation is lossless."""
    nb = K // 64
    v = rng.integers(-7, 8, size=(E, R, nb, 64))
    pos = rng.integers(0, 64, size=(E, R, nb))
    sign = rng.choice([-7, 7], size=(E, R, nb))
    np.put_along_axis(v, pos[..., None], sign[..., None], axis=3)
    j = rng.integers(-9, 2, size=(E, R, nb, 1))
    W = (v * np.exp2(j)).reshape(E, R, K)
    return _bf16(W), np.exp2(j[..., 0])


def pin_q4_format_worked_example(o):
    """Quantising the hand-worked matrix of tests/golden/q4_format.txt gives
    the bytes and scales worked out there by hand from the format statement."""
    g = read_golden("q4_format.txt")
    W = np.zeros((1, 2, 128), np.float32)
    for r, k, v in g["value"]:
        W[0, int(r), int(k)] = float(v)
    codes, scales = o.q4_quantize(_bf16(W))
    want = np.full((1, 2, 64), 0x88, np.uint8)
    for r, word, *b in g["word"]:
        want[0, int(r), 4 * int(word):4 * int(word) + 4] = [int(x, 16) for x in b]
    assert np.array_equal(codes, want)
    assert [int(x, 16) for x in g["scales"]] == scales.reshape(-1).tolist()
    assert np.array_equal(o.q4_dequant(codes, scales), W.astype(np.float64))


def pin_q4_lossless_roundtrip(o):
    """Weights exactly representable as 7-level multiples of a power of two
    per block come back unchanged, with the scale equal to that power."""
    rng = np.random.default_rng(41)
    E, R, K = 3, 5, 192  # R != K/64, so a transposed scale index cannot pass
    W, s = _exact_q4_matrix(rng, E, R, K)
    codes, scales = o.q4_quantize(W)
    assert np.array_equal(_w(scales), np.transpose(s, (0, 2, 1)))
    assert np.array_equal(o.q4_dequant(codes, scales), _w(W))


def pin_q4_error_bound(o):
    """For N(0,1) weights every dequantised weight is within half a step of the
    original (round to nearest, no clipping since |w| <= 7 s up to the bf16
    rounding of s), and s is absmax / 7 to bf16 precision."""
    rng = np.random.default_rng(42)
    E, R, K = 2, 7, 256
    W = _bf16(rng.standard_normal((E, R, K)))
    codes, scales = o.q4_quantize(W)
    Wd = o.q4_dequant(codes, scales)
    s = np.repeat(np.transpose(_w(scales), (0, 2, 1)), 64, axis=2)
    assert np.all(np.abs(Wd - _w(W)) <= 0.5 * s * (1 + 1e-12))
    amax = np.abs(_w(W)).reshape(E, R, K // 64, 64).max(-1)
    assert np.allclose(np.transpose(_w(scales), (0, 2, 1)), amax / 7.0, rtol=2.0 ** -8, atol=0)
    nib = np.concatenate([codes & 0xF, codes >> 4], axis=-1)
    assert nib.min() >= 1  # code 0 (q = -8) needs |w| > 7 s: never for these weights


def pin_q4_layer_matches_bf16_on_exact_weights(o):
    """With exactly representable expert weights the 4-bit layer equals the
    (separately pinned) bf16 layer on the same weights, slot by slot, with and
    without dropped slots."""
    rng = np.random.default_rng(43)
    T, d, f, E, k = 16, 64, 128, 4, 2
    x = _bf16(rng.standard_normal((T, d)))
    Wg = (rng.standard_normal((E, d)) / 8).astype(np.float32)
    W1, _ = _exact_q4_matrix(rng, E, f, d)
    W3, _ = _exact_q4_matrix(rng, E, f, d)
    W2, _ = _exact_q4_matrix(rng, E, d, f)
    q = [o.q4_quantize(W) for W in (W1, W3, W2)]
    for cf in (0.0, 0.5):  # dropless, and a capacity that drops slots
        r = o.route(x, Wg, k, cf=cf)
        assert (r["kept"] == 0).any() == (cf > 0)
        ref = o.layer_rows(x, W1, W3, W2, r, np.arange(T), want_h=True, want_o=True)
        got = o.layer_rows_q4(x, *q, r, np.arange(T), want_h=True, want_o=True)
        for key in ("y", "h", "o"):
            assert np.allclose(got[key], ref[key], rtol=1e-12, atol=1e-12 * np.abs(ref[key]).max()), key


Q4_PINS = [pin_q4_format_worked_example, pin_q4_lossless_roundtrip, pin_q4_error_bound,
           pin_q4_layer_matches_bf16_on_exact_weights]

ALL_PINS = ALL_PINS + Q4_PINS


# ------------------------------------------------------------ router statistics

def pin_router_stats(o):
    """The worked example's token picks experts 0 then 2; per-slot histograms
    sum to T per slot and, over the slots, to the bincount of the flattened
    top-k indices (numpy); the pair counts' margins are the first two slots'
    histograms and their diagonal is empty (the k experts are distinct)."""
    g = read_golden("worked_routing_example.txt")
    scores = np.array([float(v) for v in g["scores"]], np.float64)[None, :]
    slot, pair = o.router_stats(o.topk(scores, 2), 8)
    want = np.zeros((2, 8), np.int32)
    want[0, 0] = want[1, 2] = 1
    assert np.array_equal(slot, want) and pair[0, 2] == 1 and pair.sum() == 1
    for E, k in ((8, 2), (16, 4), (4, 1)):
        x, Wg, *_ = tiny_problem(T=50, d=32, f=32, E=E, seed=E * k)
        idx = o.topk(o.router_logits(x, Wg), k)
        slot, pair = o.router_stats(idx, E)
        assert np.all(slot.sum(1) == 50)
        assert np.array_equal(slot.sum(0), np.bincount(idx.ravel(), minlength=E))
        for j in range(k):
            assert np.array_equal(slot[j], np.bincount(idx[:, j], minlength=E))
        if k >= 2:
            assert np.array_equal(pair.sum(1), slot[0]) and np.array_equal(pair.sum(0), slot[1])
            assert np.trace(pair) == 0
            brute = np.zeros((E, E), np.int64)
            np.add.at(brute, (idx[:, 0], idx[:, 1]), 1)
            assert np.array_equal(pair, brute)


ALL_PINS = ALL_PINS + [pin_router_stats]


# --------------------------------------------------- next-best-expert fallback

def skewed_tiny(T=64, E=8, seed=4):
    """Tiny problem with two hot experts (a constant feature biases the router)."""
    x, Wg, W1, W3, W2 = tiny_problem(T=T, d=32, f=40, E=E, seed=seed)
    x = x.copy()
    Wg = Wg.copy()
    x[:, 0] = _bf16(np.ones(T))
    Wg[0, 0] += 1.5
    Wg[3 % E, 0] += 1.0
    return x, Wg, W1, W3, W2


def _brute_fallback(L, k, cf, policy):
    """Restatement of the fallback reading with numpy sorts: pass 1 as the
    capacity brute force, then each token's dropped slots (in slot order)
    move to its experts at router ranks k, k+1, ...; per expert the moved
    slots fill what pass 1 left, by full-softmax probability (ties: smaller
    token) or in token order."""
    T, E = L.shape
    order = np.array([sorted(range(E), key=lambda e: (-L[t, e], e)) for t in range(T)])
    idx = order[:, :k]
    P = np.exp(L - L.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    cap = int(np.floor(cf * T * k / E))
    S = T * k
    kept = _brute_capacity(idx.astype(np.int32), P[np.arange(T)[:, None], idx], E, cap, policy)
    expert = idx.ravel().copy()
    room = np.array([cap - sum(1 for s in range(S) if kept[s] and expert[s] == e) for e in range(E)])
    cands = {e: [] for e in range(E)}
    for t in range(T):
        m = 0
        for j in range(k):
            s = t * k + j
            if kept[s]:
                continue
            r = k + m
            m += 1
            if r < E:
                cands[order[t, r]].append((s, t, P[t, order[t, r]]))
    for e, lst in cands.items():
        if policy == 0:
            lst = sorted(lst, key=lambda c: (-c[2], c[1]))
        for s, t, _ in lst[:max(room[e], 0)]:
            kept[s] = 1
            expert[s] = e
    return expert, kept, cap


def pin_fallback_bruteforce(o):
    """The oracle's fallback equals the brute-force restatement; pass 1 is
    the plain capacity policy; a moved slot lands outside its token's top-k,
    on ranks k, k+1, ... in slot order; no expert exceeds its capacity; with
    a huge capacity nothing moves, with capacity 0 nothing is kept."""
    for (T, E, k, cf) in ((64, 8, 2, 1.0), (48, 8, 3, 0.75), (40, 4, 2, 1.25), (30, 16, 4, 1.0)):
        x, Wg, *_ = skewed_tiny(T=T, E=E, seed=T + E)
        L = o.router_logits(x, Wg)
        for base in (0, 1):
            r = o.route(x, Wg, k, cf=cf, policy=2 + base)
            expert, kept, cap = _brute_fallback(L, k, cf, base)
            assert r["cap"] == cap
            assert np.array_equal(r["kept"], kept) and np.array_equal(r["expert"].ravel(), expert), (T, E, k, base)
            plain = o.route(x, Wg, k, cf=cf, policy=base)
            stayed = r["expert"].ravel() == r["idx"].ravel()
            assert np.array_equal(plain["kept"].astype(bool), r["kept"].astype(bool) & stayed)
            moved = np.nonzero(~stayed & (r["kept"] == 1))[0]
            assert moved.size > 0
            for s in moved:
                assert r["expert"].ravel()[s] not in r["idx"][s // k]
            per = np.bincount(r["expert"].ravel()[r["kept"] == 1], minlength=E)
            assert per.max() <= cap
            assert np.array_equal(np.diff(r["offsets"]), per)
    # experts 4 and 5 with identical router rows: their logits tie exactly, and
    # a moved slot that reaches the pair takes the smaller index
    x, Wg, *_ = skewed_tiny(T=96, seed=12)
    Wg[5] = Wg[4]
    L = o.router_logits(x, Wg)
    for base in (0, 1):
        r = o.route(x, Wg, 2, cf=1.0, policy=2 + base)
        expert, kept, _ = _brute_fallback(L, 2, 1.0, base)
        assert np.array_equal(r["expert"].ravel(), expert) and np.array_equal(r["kept"], kept)
        landed = r["expert"].ravel()[(r["kept"] == 1) & (r["expert"].ravel() != r["idx"].ravel())]
        assert (landed == 4).any()
    x, Wg, *_ = skewed_tiny()
    assert not (o.route(x, Wg, 2, cf=1e9, policy=2)["expert"] != o.route(x, Wg, 2)["idx"]).any()
    assert not o.route(x, Wg, 2, cf=0.01, policy=3)["kept"].any()


def pin_fallback_layer(o):
    """With the fallback, y(t) = sum over kept slots of w_j * Expert_e(x_t),
    e the expert the slot landed on (numpy experts), the gate weight being
    the slot's own top-k weight."""
    x, Wg, W1, W3, W2 = skewed_tiny()
    r = o.route(x, Wg, 2, cf=1.0, policy=2)
    y = o.layer_rows(x, W1, W3, W2, r, np.arange(64))["y"]
    moved = 0
    for t in range(64):
        ref = np.zeros(32)
        for j in range(2):
            s = 2 * t + j
            if r["kept"][s]:
                e = r["expert"][t, j]
                moved += e != r["idx"][t, j]
                ref += r["w"][t, j] * _np_expert(_w(x[t]), W1[e], W3[e], W2[e])[1]
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-13)
    assert moved > 0


ALL_PINS = ALL_PINS + [pin_fallback_bruteforce, pin_fallback_layer]

"""The CPU oracle against its pins, and the pins against planted mistakes.

The second half compiles copies of the oracle source with one plausible
mistake each (a dropped term, a wrong sign, a swapped operand, a wrong index
or tie rule) and checks that at least one pin fails on every such copy.
"""
import os
import shutil
import tempfile

import numpy as np
import pytest

import oracle
import pins
import synth


@pytest.fixture(scope="module")
def o():
    return oracle.Oracle()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(o, pin):
    pin(o)


# The SiLU line of the bf16 and of the 4-bit expert, each with the line before
# it so that the anchor is unique.
_SILU = "b += bf16_to_double(W3e[(int64_t)n * d + i]) * xi;\n    }\n    h[n] = a / (1.0 + exp(-a)) * b;"
_SILU_Q4 = "b += q4_weight(W3c, W3s, f, d, n, i) * xi;\n    }\n    h[n] = a / (1.0 + exp(-a)) * b;"

# (description, text in moe_oracle.c, replacement) -- each is a mistake that
# a restatement of the layer could plausibly contain.
MUTANTS = [
    ("silu sign", _SILU, _SILU.replace("exp(-a)", "exp(a)")),
    ("silu dropped", _SILU, _SILU.replace("a / (1.0 + exp(-a)) * b", "a * b")),
    ("W1/W3 swapped in gate", _SILU, _SILU.replace("a / (1.0 + exp(-a)) * b", "b / (1.0 + exp(-b)) * a")),
    ("q4 silu sign", _SILU_Q4, _SILU_Q4.replace("exp(-a)", "exp(a)")),
    ("q4 combine ignores gate", "yr[c] += w[slot] * o[c];", "yr[c] += o[c];"),
    ("q4 dropped slot still added", "if (!kept[slot]) {", "if (0) {"),
    ("W2 transposed", "acc += bf16_to_double(W2e[(int64_t)c * f + n]) * h[n];",
     "acc += bf16_to_double(W2e[(int64_t)n * d + c]) * h[n];"),
    ("topk ties to larger index", "if (best < 0 || l[e] > l[best]) best = e;",
     "if (best < 0 || l[e] >= l[best]) best = e;"),
    ("gate max not subtracted consistently", "w[t * k + j] = exp(l[idx[t * k + j]] - m) / zk;",
     "w[t * k + j] = exp(l[idx[t * k + j]]) / zk;"),
    ("gate over all experts (no renormalise)", "w[t * k + j] = exp(l[idx[t * k + j]] - m) / zk;",
     "w[t * k + j] = exp(l[idx[t * k + j]] - M) / zE;"),
    ("capacity without k", "cap = (int64_t)floor(cf * (double)T * (double)k / (double)E);",
     "cap = (int64_t)floor(cf * (double)T / (double)E);"),
    ("capacity ties to larger token", "return (x->t < y->t) ? -1 : (x->t > y->t);",
     "return (x->t > y->t) ? -1 : (x->t < y->t);"),
    ("capacity keeps lowest prob", "if (x->p > y->p) return -1;\n  if (x->p < y->p) return 1;",
     "if (x->p < y->p) return -1;\n  if (x->p > y->p) return 1;"),
    ("router skips last feature", "for (int32_t i = 0; i < d; ++i)\n        acc += bf16_to_double(x[t * d + i])",
     "for (int32_t i = 0; i < d - 1; ++i)\n        acc += bf16_to_double(x[t * d + i])"),
    ("combine ignores gate", "yr[c] += w[s] * o[c];", "yr[c] += o[c];"),
    ("dropped slot still added", "if (!kept[s]) {", "if (0) {"),
    ("grouping in reverse token order", "for (int64_t s = 0; s < S; ++s) {\n      if (idx[s] != e) continue;",
     "for (int64_t s = S - 1; s >= 0; --s) {\n      if (idx[s] != e) continue;"),
    ("stats slot index swapped", "slot_counts[j * E + idx[t * k + j]] += 1;", "slot_counts[(k - 1 - j) * E + idx[t * k + j]] += 1;"),
    ("stats pair transposed", "pair_counts[idx[t * k] * E + idx[t * k + 1]] += 1;",
     "pair_counts[idx[t * k + 1] * E + idx[t * k]] += 1;"),
    ("fallback always to rank k", "int32_t r = k + moved;", "int32_t r = k;"),
    ("fallback ignores pass-1 load", "int64_t room = cap - used[e];", "int64_t room = cap;"),
    ("fallback by order under policy 0", "    if (policy == 0) qsort(list, (size_t)n, sizeof(prio_t), prio_cmp);\n    int64_t room",
     "    int64_t room"),
    ("fallback tie to larger logit index",
     "while (b >= 0 && (l[order[b]] < l[v] || (l[order[b]] == l[v] && order[b] > v))) {",
     "while (b >= 0 && (l[order[b]] < l[v] || (l[order[b]] == l[v] && order[b] < v))) {"),
    ("q4 codes in plain nibble order", "int nib = j / 2 + 4 * (j % 2);", "int nib = j;"),
    ("q4 high and low nibble swapped", "*shift = 4 * (nib % 2);", "*shift = 4 * (1 - nib % 2);"),
    ("q4 scales read row-major", "bf16_to_double(scales_e[(k / 64) * R + r]);",
     "bf16_to_double(scales_e[r * (K / 64) + k / 64]);"),
    ("q4 code offset 7", "return (double)(code - 8) * bf16_to_double", "return (double)(code - 7) * bf16_to_double"),
    ("q4 scale absmax / 8", "float s = q4_bf16_round(amax / 7.0f);", "float s = q4_bf16_round(amax / 8.0f);"),
    ("q4 truncating round", "float v = nearbyintf((float)bf16_to_double(wr[i]) / s);",
     "float v = truncf((float)bf16_to_double(wr[i]) / s);"),
    ("q4 W2 read with W1 shape", "acc += q4_weight(W2c, W2s, d, f, c, n) * h[n];",
     "acc += q4_weight(W2c, W2s, f, d, c % f, n % d) * h[n];"),
    ("q4 W3 scales from W1", "b += q4_weight(W3c, W3s, f, d, n, i) * xi;", "b += q4_weight(W3c, W1s, f, d, n, i) * xi;"),
    ("capacity rounded up", "cap = (int64_t)floor(cf * (double)T * (double)k / (double)E);",
     "cap = (int64_t)ceil(cf * (double)T * (double)k / (double)E);"),
    ("topk picks the smallest logit", "if (best < 0 || l[e] > l[best]) best = e;",
     "if (best < 0 || l[e] < l[best]) best = e;"),
    ("topk may repeat an expert", "taken |= (idx[t * k + q] == e);", "taken |= 0;"),
    ("probability normalised over the top k", "p[t * k + j] = exp(l[idx[t * k + j]] - M) / zE;",
     "p[t * k + j] = exp(l[idx[t * k + j]] - m) / zk;"),
    ("router reads Wg transposed", "(double)Wg[(int64_t)e * d + i]", "(double)Wg[(int64_t)i * E + e]"),
    ("router writes logits to the next expert", "logits[t * E + e] = acc;", "logits[t * E + (e + 1) % E] = acc;"),
    ("swiglu sum instead of product", _SILU, _SILU.replace("a / (1.0 + exp(-a)) * b", "a / (1.0 + exp(-a)) + b")),
    ("up projection from W1", "b += bf16_to_double(W3e[(int64_t)n * d + i]) * xi;",
     "b += bf16_to_double(W1e[(int64_t)n * d + i]) * xi;"),
    ("layer runs every slot on the first choice's expert", "int64_t e = idx[s];", "int64_t e = idx[t * k];"),
    ("capacity keeps the end of the priority list", "for (int64_t r = 0; r < n && r < cap; ++r) kept[list[r].s] = 1;",
     "for (int64_t r = 0; r < n && r < cap; ++r) kept[list[n - 1 - r].s] = 1;"),
    ("capacity keeps one slot fewer", "for (int64_t r = 0; r < n && r < cap; ++r) kept[list[r].s] = 1;",
     "for (int64_t r = 0; r < n && r < cap - 1; ++r) kept[list[r].s] = 1;"),
    ("capacity lists other experts' slots", "if (idx[s] == e) {\n        list[n].p = p[s];",
     "if (idx[s] != e) {\n        list[n].p = p[s];"),
    ("offsets hold starts, not ends", "offsets[e + 1] = (int32_t)row;", "offsets[e + 1] = (int32_t)row - kept_counts[e];"),
    ("dropped slot gets row 0", "slot_pos[s] = -1;", "slot_pos[s] = 0;"),
    ("fallback keeps the old expert's probability", "cand_p[s] = exp(l[order[r]] - M) / zE;", "cand_p[s] = p[s];"),
    ("fallback skips rank k", "int32_t r = k + moved;", "int32_t r = k + 1 + moved;"),
    ("fallback moves kept slots too", "if (kept[s]) continue;", "if (0) continue;"),
    ("fallback ignores the capacity", "int64_t room = cap - used[e];", "int64_t room = n;"),
    ("fallback router order ascending", "while (b >= 0 && (l[order[b]] < l[v] ||", "while (b >= 0 && (l[order[b]] > l[v] ||"),
    ("q4 scale not rounded to bf16", "float s = q4_bf16_round(amax / 7.0f);", "float s = amax / 7.0f;"),
    ("q4 bf16 rounding truncates", "u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;", "u = u & 0xFFFF0000u;"),
    ("q4 absmax without magnitude", "float v = fabsf((float)bf16_to_double(wr[i]));",
     "float v = (float)bf16_to_double(wr[i]);"),
    ("q4 absmax over half the block", "for (int i = 0; i < 64; ++i) {\n          float v = fabsf",
     "for (int i = 0; i < 32; ++i) {\n          float v = fabsf"),
    ("q4 wrong byte within the word", "*byte = g * 4 + nib / 2;", "*byte = g * 4 + nib % 4;"),
    ("q4 scale stored for the next row", "scales[((int64_t)e * nb + b) * R + r] = (uint16_t)(sb >> 16);",
     "scales[((int64_t)e * nb + b) * R + (r + 1) % R] = (uint16_t)(sb >> 16);"),
    ("q4 dequantiser ignores the expert's scale offset", "const uint16_t *se = scales + (int64_t)e * (K / 64) * R;",
     "const uint16_t *se = scales;"),
]
# Not listed because they cannot change any output for bf16 weights (the
# first while absmax / 7 is a normal fp32 number):
# * rounding the scale's ties upward instead of to even: absmax / 7 with an
#   8-bit absmax mantissa is never a bf16 tie (past its 8th bit the quotient
#   repeats the bits of a multiple of 1/7, never exactly 1000...0);
# * clamping codes at -7 instead of -8: |w / s| <= 7 (1 + 2^-8) < 7.5, so the
#   lower clamp is never reached.


@pytest.mark.parametrize("desc,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(desc, old, new):
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {desc}"
    tmpdir = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        msrc = os.path.join(tmpdir, "mutant.c")
        with open(msrc, "w") as fh:
            fh.write(src.replace(old, new))
        lib = oracle._bind(oracle.build(force=True, src=msrc, out=os.path.join(tmpdir, "libm.so")))
        m = oracle.Oracle(lib)
        caught = []
        for pin in pins.ALL_PINS:
            try:
                pin(m)
            except AssertionError:
                caught.append(pin.__name__)
            except Exception as exc:  # a crash also counts as caught
                caught.append(f"{pin.__name__}:{type(exc).__name__}")
        assert caught, f"no pin caught the planted mistake: {desc}"
    finally:
        shutil.rmtree(tmpdir, ignore_errors=True)


def test_generator_definition():
    """The input generator follows its stated definition: splitmix64 words,
    Box-Muller, round-to-nearest-even bf16; moments of a large draw."""
    G = 0x9E3779B97F4A7C15
    M = (1 << 64) - 1

    def mix(z):
        z ^= z >> 30
        z = (z * 0xBF58476D1CE4E5B9) & M
        z ^= z >> 27
        z = (z * 0x94D049BB133111EB) & M
        return z ^ (z >> 31)

    seed, tid = 3, 4
    base = mix(mix((seed + G) & M) ^ ((tid * 0xD1B54A32D192ED03) & M))
    want = [mix((base + (n + 1) * G) & M) for n in range(6)]
    assert synth.words(seed, tid, 6).tolist() == want
    import math
    u1 = ((want[0] >> 11) + 1) * 2.0 ** -53
    u2 = (want[1] >> 11) * 2.0 ** -53
    z0 = math.sqrt(-2 * math.log(u1)) * math.cos(2 * math.pi * u2)
    v = synth.normal_f32(seed, tid, 1)
    assert abs(float(v[0]) - z0) <= 1e-6 * max(1.0, abs(z0))
    b = synth.normal_bf16(seed, tid, 1)
    assert abs(float(synth.bf16_to_f32(b)[0]) - z0) <= abs(z0) * 2.0 ** -8
    big = synth.normal_f32(0, 9, 1 << 20).astype(np.float64)
    assert abs(big.mean()) < 5e-3 and abs(big.std() - 1.0) < 5e-3
    # bf16 rounding is nearest-even
    assert synth.f32_to_bf16(np.array([1.0 + 2 ** -8], np.float32))[0] == 0x3F80
    assert synth.f32_to_bf16(np.array([1.0 + 3 * 2 ** -8], np.float32))[0] == 0x3F82


def test_skew_recipe_share():
    """The skewed workload's constant feature and router bias send close to
    40 % of top-2 slots to expert 0 (sampled on 2048 tokens)."""
    wl = synth.workload("skew", T=2048)
    wl.generate(weights=False)
    o = oracle.Oracle()
    idx = o.topk(o.router_logits(wl.x, wl.Wg), 2)
    share = float((idx == 0).sum()) / idx.size
    assert 0.37 < share < 0.43, share

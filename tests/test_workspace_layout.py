"""The workspace layout as stated for callers, against moe_workspace_size.

Regions, in order, each starting on a 256-byte boundary:
  control: status word, tile ticket and two GEMM tile counters (16 bytes);
           counts [E] int32; with the next-best fallback, three [E] int32
           counters; look-back words [ceil(S / 64), E] uint32
  capacity thresholds [E] uint64
  split-K partials [splits, S, d] fp32 (streaming schedule and 4-bit only)
  topk_idx, topk_w, topk_p [S]; offsets [E + 1]; slot_pos, perm_slot [S]
  x_perm [S, d], h [S, f], y_perm [S, d] bf16
  x and y staging [T, d] bf16 (host-buffer entry point)
  with the next-best fallback: next ranks [S] int32 and probabilities [S]
  fp32, two key arrays [S] uint64, candidates and landed experts [S] int32,
  second thresholds [E] uint64
with S = T * k.  The split count of the streaming schedule is a tuning
choice, so only its form (a whole number of [S, d] fp32 planes, 1 to 16)
is checked.
"""
import pytest

A = 256


def al(v):
    return (v + A - 1) // A * A


def expected(T, d, f, E, k, fallback=False):
    S = T * k
    o = al(16) + al(4 * E)
    if fallback:
        o += al(3 * 4 * E)
    o += al(4 * ((S + 63) // 64) * E)
    o += al(8 * E)
    o += 3 * al(4 * S) + al(4 * (E + 1)) + 2 * al(4 * S)
    o += al(2 * S * d) + al(2 * S * f) + al(2 * S * d)
    o += 2 * al(2 * T * d)
    if fallback:
        o += 2 * al(4 * S) + 2 * al(8 * S) + 2 * al(4 * S) + al(8 * E)
    return o


@pytest.fixture(scope="module")
def moe():
    from sparse_mixture_experts_13_b200 import build as b
    b.build()
    import sparse_mixture_experts_13_b200 as m
    return m


@pytest.mark.parametrize("T,d,f,E,k,variant,cf,policy", [
    (300, 128, 448, 8, 2, 1, 0.0, 0),          # CTA-pair schedule
    (4096, 4096, 14336, 8, 2, 0, 0.0, 0),      # prefill: AUTO picks the tiled schedule
    (200, 256, 512, 16, 4, 3, 0.0, 0),         # single-CTA tiles
    (8192, 4096, 14336, 8, 2, 0, 1.25, 0),     # capacity by probability: same regions
    (1000, 128, 256, 8, 2, 1, 1.25, 2),        # next-best fallback adds its arrays
    (777, 64, 64, 32, 8, 1, 0.5, 3),
])
def test_tiled_layout(moe, T, d, f, E, k, variant, cf, policy):
    sh = moe.make_shape(T, d, f, E, k, cf, policy, variant)
    assert moe.moe_workspace_size(sh) == expected(T, d, f, E, k, fallback=cf > 0 and policy >= 2)


def _splits(extra, S, d):
    """Number of [S, d] fp32 planes that `extra` bytes hold, or None."""
    for sp in range(1, 17):
        if al(4 * sp * S * d) == extra:
            return sp
    return None


@pytest.mark.parametrize("T,d,f", [(16, 4096, 14336), (1, 4096, 14336), (2, 4096, 14336), (128, 128, 448),
                                   (64, 256, 512)])
def test_streaming_layout_adds_splitk_planes(moe, T, d, f):
    """The streaming schedule adds the down projection's split-K planes
    [splits, S, d] fp32; at one or two Mixtral tokens (2 or 4 experts' tiles
    fill the last wave of 148 SMs poorly) the gate/up projection is split 2
    ways along K too, adding [2, S, 2 f] fp32 partials."""
    sh = moe.make_shape(T, d, f)                 # AUTO: streaming schedule for T <= 128
    extra = moe.moe_workspace_size(sh) - expected(T, d, f, 8, 2)
    if T <= 2 and f == 14336:
        extra -= al(4 * 2 * T * 2 * 2 * f)
    assert _splits(extra, T * 2, d) is not None, extra


@pytest.mark.parametrize("T", [16, 32, 33, 64, 65, 88, 89, 300])
def test_q4_layout_always_has_splitk_planes(moe, T):
    """The 4-bit layout adds split-K planes and, for token tiles of 16 and 32
    (the integer-MMA kernels; the tile is 16 while the mean slots per expert
    fit it, 32 up to a mean of 22, else twice the mean: for 8 experts and
    top-2, 16 up to T = 64, 32 up to 88, then 64), the quantised activations
    as their tiled token
    operand and their scales [S] fp32 at the end.  The operand
    holds, per token tile (at most S / bn + E of them) and stage of ks inputs
    (256 for 16-token tiles, 128 for 32), the high and low bytes of the
    tile's bn rows: 2 bn x ks bytes."""
    sh = moe.make_shape(T, 4096, 14336)
    extra = moe.moe_workspace_size_q4(sh) - expected(T, 4096, 14336, 8, 2)
    S = T * 2
    mean = -(-S // 8)
    bn = 16 if mean <= 16 else 32 if mean <= 22 else -(-2 * mean // 16) * 16    # token tile
    if bn <= 32:
        ks = 256 if bn == 16 else 128
        tiles = -(-S // bn) + 8
        extra -= al(tiles * -(-14336 // ks) * 2 * bn * ks) + al(4 * S)
    assert _splits(extra, S, 4096) is not None, extra


def test_quoted_sizes(moe):
    """The workspace sizes quoted for the Mixtral-shaped workloads."""
    mb = lambda T: moe.moe_workspace_size(moe.make_shape(T, 4096, 14336)) / 1e6
    assert round(mb(16), 1) == 3.8
    assert round(mb(4096)) == 436
    assert round(mb(32768) / 1e3, 1) == 3.5

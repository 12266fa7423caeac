"""Router statistics through the C ABI against the oracle, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mixture_experts_13_b200 as moe
    import gpu_harness as H
else:  # collected on CPU hosts, never run there
    moe = H = None


@pytest.fixture(scope="module")
def o():
    return oracle.Oracle()


def gpu_stats(sh, idx_dev, E, k, pair=True, accumulate=0, slot=None, pr=None):
    slot = torch.zeros(k, E, dtype=torch.int32, device="cuda") if slot is None else slot
    pr = (torch.zeros(E, E, dtype=torch.int32, device="cuda") if pr is None else pr) if pair else None
    moe.check(moe.moe_router_stats(sh, idx_dev, slot, pr, accumulate), "router_stats")
    torch.cuda.synchronize()
    return slot, pr


@pytest.mark.parametrize("T,E,k", [(64, 8, 2), (1, 8, 2), (777, 16, 4), (300, 32, 8), (200, 4, 1), (4096, 8, 2)])
def test_router_stats_match_oracle(o, T, E, k):
    wl = synth.Workload(f"st{T}", T, 128, 192, E=E, k=k, seed=T + E).generate(weights=False)
    dev = H.Device.__new__(H.Device)
    dev.wl, dev.x, dev.Wg = wl, H.to_dev_bf16(wl.x), torch.from_numpy(wl.Wg).cuda()
    sh = dev.shape(0)
    S = T * k
    idx = torch.empty(S, dtype=torch.int32, device="cuda")
    w = torch.empty(S, dtype=torch.float32, device="cuda")
    p = torch.empty(S, dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    moe.check(moe.moe_router_topk(sh, dev.x, dev.Wg, None, idx, w, p, counts), "router")
    slot, pr = gpu_stats(sh, idx, E, k, pair=k >= 2)
    ref_slot, ref_pair = o.router_stats(idx.cpu().numpy().reshape(T, k), E)
    assert np.array_equal(slot.cpu().numpy(), ref_slot)
    if k >= 2:
        assert np.array_equal(pr.cpu().numpy(), ref_pair)
    # the slot histograms add up to the layer's counts
    assert np.array_equal(slot.cpu().numpy().sum(0), counts.cpu().numpy())
    # accumulate: a second call adds the same histograms again
    slot2, pr2 = gpu_stats(sh, idx, E, k, pair=k >= 2, accumulate=1, slot=slot.clone(),
                           pr=pr.clone() if pr is not None else None)
    assert np.array_equal(slot2.cpu().numpy(), 2 * ref_slot)


def test_router_stats_layer_table_and_clear():
    """Rows of a [layers, E] activation table filled from the layer's counts
    and per-slot histograms; T == 0 with accumulate = 0 only clears."""
    E, k = 8, 2
    idx = torch.tensor([[0, 2], [2, 0], [0, 2], [7, 1]], dtype=torch.int32, device="cuda").reshape(-1)
    sh = moe.make_shape(4, 128, 192, E, k)
    table = torch.zeros(3, k, E, dtype=torch.int32, device="cuda")
    moe.check(moe.moe_router_stats(sh, idx, table[1], None, 0), "stats")
    torch.cuda.synchronize()
    t = table.cpu().numpy()
    assert not t[0].any() and not t[2].any()
    assert t[1, 0].tolist() == [2, 0, 1, 0, 0, 0, 0, 1] and t[1, 1].tolist() == [1, 1, 2, 0, 0, 0, 0, 0]
    assert int(np.argmax(t[1, 0])) == 0 and int(np.argmax(t[1, 1])) == 2  # most common expert per position
    sh0 = moe.make_shape(0, 128, 192, E, k)
    moe.check(moe.moe_router_stats(sh0, None, table[1], None, 0), "stats clear")
    torch.cuda.synchronize()
    assert not table.cpu().numpy().any()

"""Expert-parallel MoE layer: the experts are split over `world` ranks, the
tokens are dispatched to the ranks that own their experts and the results
come back (source: "How Mixtral 8x7B uses mixture of experts", "Tensor
parallelism vs expert parallelism", expert_parallel_forward).

The computation is the library's: ``moe_router_topk``, ``moe_ep_plan``,
``moe_ep_dispatch`` (grouping fused with the dispatch: token rows are stored
straight into the owner's receive buffer), ``moe_grouped_swiglu`` on the
owner, and ``moe_ep_combine`` (combine fused with the return: result rows are
read from the owner's buffer).  This module only allocates buffers and
orders the steps.

Two drivers:
* ``ep_forward_emulated`` runs every rank's steps on one GPU, the ranks'
  buffers being ordinary device allocations and the "peer" pointers plain
  device pointers; the steps of all ranks run phase by phase in stream order,
  so no kernel waits on another.  It checks the dispatch, the owners' GEMMs
  and the combine on a single device.
* ``EPLayer`` is the one-process-per-GPU form: counts are all-gathered with
  NCCL, the receive buffers live in symmetric memory so that every rank holds
  the others' pointers, and ``torch.distributed`` barriers separate the
  dispatch, the expert GEMMs and the combine.
"""
from __future__ import annotations

import torch

from . import _lib


def _check(st, what):
    _lib.check(st, what)


def _ptrs(tensors, device) -> torch.Tensor:
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


def ep_forward_emulated(xs, Wg, W1, W3, W2, world: int, k: int = 2, capacity_factor: float = 0.0,
                        drop_policy: int = _lib.MOE_DROP_BY_PROB, info: dict | None = None):
    """Expert-parallel forward of `world` emulated ranks on one GPU.

    xs: list of `world` bf16 [T_r, d] token batches; Wg fp32 [E, d]; W1, W3
    [E, f, d] and W2 [E, d, f] bf16 (rank o uses experts o*E/world ..).
    With capacity_factor > 0 the ranks' tokens are one batch (their
    concatenation) and each owner keeps its experts' slots under the capacity
    (moe_ep_dispatch_cap, moe_ep_select, moe_ep_combine_cap).
    Returns (list of y [T_r, d], list of topk_idx [T_r*k], list of counts [E]);
    `info`, if given, receives the routers' probabilities, ret_row of every
    rank and row_map of every owner.
    """
    dev = xs[0].device
    E, f, d = W1.shape
    assert E % world == 0 and len(xs) == world
    epr = E // world
    cap_mode = capacity_factor > 0
    cu = lambda *shape, dt: torch.empty(*shape, dtype=dt, device=dev)
    # 1. routers
    shapes = [_lib.make_shape(x.shape[0], d, f, E, k, capacity_factor, drop_policy) for x in xs]
    idx, w, probs, counts = [], [], [], []
    for r, x in enumerate(xs):
        T = x.shape[0]
        i, ww, p, c = cu(T * k, dt=torch.int32), cu(T * k, dt=torch.float32), cu(T * k, dt=torch.float32), \
            cu(E, dt=torch.int32)
        _check(_lib.moe_router_topk(shapes[r], x, Wg, None, i, ww, p, c), "moe_router_topk")
        idx.append(i)
        w.append(ww)
        probs.append(p)
        counts.append(c)
    # 2. all-gather of the counts
    counts_all = torch.stack(counts).contiguous()
    # 3. plans; receive buffers sized for every slot of every rank
    rows = sum(x.shape[0] for x in xs) * k
    x_recv = [cu(rows, d, dt=torch.bfloat16) for _ in range(world)]
    y_recv = [cu(rows, d, dt=torch.bfloat16) for _ in range(world)]
    h_recv = [cu(rows, f, dt=torch.bfloat16) for _ in range(world)]
    peer_x, peer_y = _ptrs(x_recv, dev), _ptrs(y_recv, dev)
    recv_off = [cu(E, dt=torch.int32) for _ in range(world)]
    owner_off = [cu(epr + 1, dt=torch.int32) for _ in range(world)]
    for r in range(world):
        _check(_lib.moe_ep_plan(counts_all, E, r, world, recv_off[r], owner_off[r]), "moe_ep_plan")
    if cap_mode:
        keys = [cu(max(rows, 1), dt=torch.int64) for _ in range(world)]
        row_map = [cu(max(rows, 1), dt=torch.int32) for _ in range(world)]
        x_kept = [cu(rows, d, dt=torch.bfloat16) for _ in range(world)]
        kept_off = [cu(epr + 1, dt=torch.int32) for _ in range(world)]
        peer_keys, peer_map = _ptrs(keys, dev), _ptrs(row_map, dev)
    # 4. dispatch
    ret_row = []
    for r, x in enumerate(xs):
        rr = cu(x.shape[0] * k, dt=torch.int32)
        n = _lib.moe_workspace_size(shapes[r])
        ws = cu(n, dt=torch.uint8)
        if cap_mode:
            _check(_lib.moe_ep_dispatch_cap(shapes[r], world, r, counts_all, x, idx[r], probs[r], counts[r],
                                            recv_off[r], peer_x, peer_keys, rr, ws, n), "moe_ep_dispatch_cap")
        else:
            _check(_lib.moe_ep_dispatch(shapes[r], world, x, idx[r], counts[r], recv_off[r], peer_x, rr, ws, n),
                   "moe_ep_dispatch")
        ret_row.append(rr)
    # 5. owners: the capacity (with one) and the expert GEMMs
    osh = _lib.make_shape(rows, d, f, epr, 1)
    n = _lib.moe_workspace_size(osh)
    for o in range(world):
        ws = cu(n, dt=torch.uint8)
        sl = slice(o * epr, (o + 1) * epr)
        a_in, a_off = x_recv[o], owner_off[o]
        if cap_mode:
            _check(_lib.moe_ep_select(shapes[0], world, counts_all, owner_off[o], keys[o], x_recv[o], x_kept[o],
                                      kept_off[o], row_map[o]), "moe_ep_select")
            a_in, a_off = x_kept[o], kept_off[o]
        _check(_lib.moe_grouped_swiglu(osh, a_in, a_off, W1[sl].contiguous(), W3[sl].contiguous(),
                                       W2[sl].contiguous(), h_recv[o], y_recv[o], ws, n), "moe_grouped_swiglu")
    # 6. combine
    ys = []
    for r, x in enumerate(xs):
        y = cu(x.shape[0], d, dt=torch.bfloat16)
        if cap_mode:
            _check(_lib.moe_ep_combine_cap(shapes[r], world, idx[r], w[r], ret_row[r], peer_map, peer_y, y),
                   "moe_ep_combine_cap")
        else:
            _check(_lib.moe_ep_combine(shapes[r], world, idx[r], w[r], ret_row[r], peer_y, y), "moe_ep_combine")
        ys.append(y)
    if info is not None:
        info.update(p=probs, ret_row=ret_row, row_map=row_map if cap_mode else None, epr=epr)
    return ys, idx, counts


class EPLayer:
    """One rank of an expert-parallel layer, one process per GPU.

    Holds this rank's experts (E / world of them) and receive buffers in
    symmetric memory for up to `max_tokens` tokens per rank.  ``forward``
    runs the layer on this rank's tokens; every rank must call it with the
    same sequence of layers (it contains collectives).
    """

    def __init__(self, Wg, W1_local, W3_local, W2_local, E: int, k: int, max_tokens: int, group=None,
                 capacity_factor: float = 0.0, drop_policy: int = _lib.MOE_DROP_BY_PROB):
        import os
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm_mem
        # The kernels use plain peer loads and stores; the buffers need no
        # NVLink multicast object (none is bound to them).
        os.environ.setdefault("TORCH_SYMM_MEM_DISABLE_MULTICAST", "1")
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        assert E % self.world == 0 and W1_local.shape[0] == E // self.world
        self.Wg, self.W1, self.W3, self.W2 = Wg, W1_local, W3_local, W2_local
        self.E, self.k = E, k
        self.epr, self.f, self.d = W1_local.shape
        dev = Wg.device
        self.rows = max_tokens * k * self.world
        self.x_recv = symm_mem.empty(self.rows, self.d, dtype=torch.bfloat16, device=dev)
        self.y_recv = symm_mem.empty(self.rows, self.d, dtype=torch.bfloat16, device=dev)
        g = group or dist.group.WORLD
        hx = symm_mem.rendezvous(self.x_recv, group=g)
        hy = symm_mem.rendezvous(self.y_recv, group=g)
        # the tensor may sit at an offset inside its symmetric buffer; every
        # rank's copy sits at the same offset
        ox = self.x_recv.data_ptr() - hx.buffer_ptrs[self.rank]
        oy = self.y_recv.data_ptr() - hy.buffer_ptrs[self.rank]
        self.peer_x = torch.tensor([p_ + ox for p_ in hx.buffer_ptrs], dtype=torch.int64, device=dev)
        self.peer_y = torch.tensor([p_ + oy for p_ in hy.buffer_ptrs], dtype=torch.int64, device=dev)
        self._handles = (hx, hy)
        self.h_recv = torch.empty(self.rows, self.f, dtype=torch.bfloat16, device=dev)
        self.capacity_factor, self.drop_policy = capacity_factor, drop_policy
        if capacity_factor > 0:
            # the owner's key buffer and row map are written / read by the
            # other ranks, so they live in symmetric memory too
            self.keys = symm_mem.empty(self.rows, dtype=torch.int64, device=dev)
            self.row_map = symm_mem.empty(self.rows, dtype=torch.int32, device=dev)
            hk = symm_mem.rendezvous(self.keys, group=g)
            hm = symm_mem.rendezvous(self.row_map, group=g)
            ok_ = self.keys.data_ptr() - hk.buffer_ptrs[self.rank]
            om = self.row_map.data_ptr() - hm.buffer_ptrs[self.rank]
            self.peer_keys = torch.tensor([p_ + ok_ for p_ in hk.buffer_ptrs], dtype=torch.int64, device=dev)
            self.peer_map = torch.tensor([p_ + om for p_ in hm.buffer_ptrs], dtype=torch.int64, device=dev)
            self._handles = self._handles + (hk, hm)
            self.x_kept = torch.empty(self.rows, self.d, dtype=torch.bfloat16, device=dev)
            self.kept_off = torch.empty(self.epr + 1, dtype=torch.int32, device=dev)
        self.owner_shape = _lib.make_shape(self.rows, self.d, self.f, self.epr, 1)
        self.owner_ws = torch.empty(_lib.moe_workspace_size(self.owner_shape), dtype=torch.uint8, device=dev)

    def forward(self, x: torch.Tensor, events=None) -> torch.Tensor:
        """`events`, if given, is a list of 5 CUDA events recorded on the
        current stream before the router and after the plan, the dispatch,
        the owner's GEMMs and the combine (phase times for benchmarks)."""
        dist, dev = self.dist, x.device
        mark = (lambda i: events[i].record()) if events is not None else (lambda i: None)
        mark(0)
        T, d, E, k = x.shape[0], self.d, self.E, self.k
        cap_mode = self.capacity_factor > 0
        sh = _lib.make_shape(T, d, self.f, E, k, self.capacity_factor, self.drop_policy)
        cu = lambda *shape, dt: torch.empty(*shape, dtype=dt, device=dev)
        idx, w, p, counts = cu(T * k, dt=torch.int32), cu(T * k, dt=torch.float32), cu(T * k, dt=torch.float32), \
            cu(E, dt=torch.int32)
        _check(_lib.moe_router_topk(sh, x, self.Wg, None, idx, w, p, counts), "moe_router_topk")
        counts_all = cu(self.world * E, dt=torch.int32)
        dist.all_gather_into_tensor(counts_all, counts, group=self.group)
        recv_off, owner_off = cu(E, dt=torch.int32), cu(self.epr + 1, dt=torch.int32)
        _check(_lib.moe_ep_plan(counts_all, E, self.rank, self.world, recv_off, owner_off), "moe_ep_plan")
        self.last_counts_all = counts_all
        mark(1)
        ret_row = cu(T * k, dt=torch.int32)
        n = _lib.moe_workspace_size(sh)
        ws = cu(n, dt=torch.uint8)
        if cap_mode:
            _check(_lib.moe_ep_dispatch_cap(sh, self.world, self.rank, counts_all, x, idx, p, counts, recv_off,
                                            self.peer_x, self.peer_keys, ret_row, ws, n), "moe_ep_dispatch_cap")
        else:
            _check(_lib.moe_ep_dispatch(sh, self.world, x, idx, counts, recv_off, self.peer_x, ret_row, ws, n),
                   "moe_ep_dispatch")
        mark(2)
        dist.barrier(group=self.group)  # every rank's rows (and keys) have landed
        a_in, a_off = self.x_recv, owner_off
        if cap_mode:
            _check(_lib.moe_ep_select(sh, self.world, counts_all, owner_off, self.keys, self.x_recv, self.x_kept,
                                      self.kept_off, self.row_map), "moe_ep_select")
            a_in, a_off = self.x_kept, self.kept_off
        _check(_lib.moe_grouped_swiglu(self.owner_shape, a_in, a_off, self.W1, self.W3, self.W2,
                                       self.h_recv, self.y_recv, self.owner_ws, self.owner_ws.numel()),
               "moe_grouped_swiglu")
        mark(3)
        dist.barrier(group=self.group)  # every owner's results (and row map) are written
        y = cu(T, d, dt=torch.bfloat16)
        if cap_mode:
            _check(_lib.moe_ep_combine_cap(sh, self.world, idx, w, ret_row, self.peer_map, self.peer_y, y),
                   "moe_ep_combine_cap")
        else:
            _check(_lib.moe_ep_combine(sh, self.world, idx, w, ret_row, self.peer_y, y), "moe_ep_combine")
        mark(4)
        dist.barrier(group=self.group)  # the buffers may be reused by the next call
        return y


def ep_plan_host(counts_all, rank: int, world: int):
    """The plan of moe_ep_plan on the host (lists): recv_off [E] of `rank` as
    a source and owner_off [E/world + 1] of `rank` as an owner."""
    E = len(counts_all[0])
    epr = E // world
    recv_off, owner_off = [0] * E, [0] * (epr + 1)
    for o in range(world):
        row = 0
        for l in range(epr):
            e = o * epr + l
            if o == rank:
                owner_off[l] = row
            for r in range(world):
                if r == rank:
                    recv_off[e] = row
                row += counts_all[r][e]
        if o == rank:
            owner_off[epr] = row
    return recv_off, owner_off

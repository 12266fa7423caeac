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


def ep_forward_emulated(xs, Wg, W1, W3, W2, world: int, k: int = 2):
    """Expert-parallel forward of `world` emulated ranks on one GPU.

    xs: list of `world` bf16 [T_r, d] token batches; Wg fp32 [E, d]; W1, W3
    [E, f, d] and W2 [E, d, f] bf16 (rank o uses experts o*E/world ..).
    Returns (list of y [T_r, d], list of topk_idx [T_r*k], list of counts [E]).
    """
    dev = xs[0].device
    E, f, d = W1.shape
    assert E % world == 0 and len(xs) == world
    epr = E // world
    cu = lambda *shape, dt: torch.empty(*shape, dtype=dt, device=dev)
    # 1. routers
    shapes = [_lib.make_shape(x.shape[0], d, f, E, k) for x in xs]
    idx, w, counts = [], [], []
    for r, x in enumerate(xs):
        T = x.shape[0]
        i, ww, p, c = cu(T * k, dt=torch.int32), cu(T * k, dt=torch.float32), cu(T * k, dt=torch.float32), \
            cu(E, dt=torch.int32)
        _check(_lib.moe_router_topk(shapes[r], x, Wg, None, i, ww, p, c), "moe_router_topk")
        idx.append(i)
        w.append(ww)
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
    # 4. dispatch
    ret_row = []
    for r, x in enumerate(xs):
        rr = cu(x.shape[0] * k, dt=torch.int32)
        n = _lib.moe_workspace_size(shapes[r])
        ws = cu(n, dt=torch.uint8)
        _check(_lib.moe_ep_dispatch(shapes[r], world, x, idx[r], counts[r], recv_off[r], peer_x, rr, ws, n),
               "moe_ep_dispatch")
        ret_row.append(rr)
    # 5. owners' expert GEMMs on their receive buffers
    osh = _lib.make_shape(rows, d, f, epr, 1)
    n = _lib.moe_workspace_size(osh)
    for o in range(world):
        ws = cu(n, dt=torch.uint8)
        sl = slice(o * epr, (o + 1) * epr)
        _check(_lib.moe_grouped_swiglu(osh, x_recv[o], owner_off[o], W1[sl].contiguous(), W3[sl].contiguous(),
                                       W2[sl].contiguous(), h_recv[o], y_recv[o], ws, n), "moe_grouped_swiglu")
    # 6. combine
    ys = []
    for r, x in enumerate(xs):
        y = cu(x.shape[0], d, dt=torch.bfloat16)
        _check(_lib.moe_ep_combine(shapes[r], world, idx[r], w[r], ret_row[r], peer_y, y), "moe_ep_combine")
        ys.append(y)
    return ys, idx, counts


class EPLayer:
    """One rank of an expert-parallel layer, one process per GPU.

    Holds this rank's experts (E / world of them) and receive buffers in
    symmetric memory for up to `max_tokens` tokens per rank.  ``forward``
    runs the layer on this rank's tokens; every rank must call it with the
    same sequence of layers (it contains collectives).
    """

    def __init__(self, Wg, W1_local, W3_local, W2_local, E: int, k: int, max_tokens: int, group=None):
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm_mem
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
        self.owner_shape = _lib.make_shape(self.rows, self.d, self.f, self.epr, 1)
        self.owner_ws = torch.empty(_lib.moe_workspace_size(self.owner_shape), dtype=torch.uint8, device=dev)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        dist, dev = self.dist, x.device
        T, d, E, k = x.shape[0], self.d, self.E, self.k
        sh = _lib.make_shape(T, d, self.f, E, k)
        cu = lambda *shape, dt: torch.empty(*shape, dtype=dt, device=dev)
        idx, w, p, counts = cu(T * k, dt=torch.int32), cu(T * k, dt=torch.float32), cu(T * k, dt=torch.float32), \
            cu(E, dt=torch.int32)
        _check(_lib.moe_router_topk(sh, x, self.Wg, None, idx, w, p, counts), "moe_router_topk")
        counts_all = cu(self.world * E, dt=torch.int32)
        dist.all_gather_into_tensor(counts_all, counts, group=self.group)
        recv_off, owner_off = cu(E, dt=torch.int32), cu(self.epr + 1, dt=torch.int32)
        _check(_lib.moe_ep_plan(counts_all, E, self.rank, self.world, recv_off, owner_off), "moe_ep_plan")
        ret_row = cu(T * k, dt=torch.int32)
        n = _lib.moe_workspace_size(sh)
        ws = cu(n, dt=torch.uint8)
        _check(_lib.moe_ep_dispatch(sh, self.world, x, idx, counts, recv_off, self.peer_x, ret_row, ws, n),
               "moe_ep_dispatch")
        dist.barrier(group=self.group)  # every rank's rows have landed
        _check(_lib.moe_grouped_swiglu(self.owner_shape, self.x_recv, owner_off, self.W1, self.W3, self.W2,
                                       self.h_recv, self.y_recv, self.owner_ws, self.owner_ws.numel()),
               "moe_grouped_swiglu")
        dist.barrier(group=self.group)  # every owner's results are written
        y = cu(T, d, dt=torch.bfloat16)
        _check(_lib.moe_ep_combine(sh, self.world, idx, w, ret_row, self.peer_y, y), "moe_ep_combine")
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

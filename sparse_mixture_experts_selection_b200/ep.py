"""Expert parallelism: the routed experts are split over W ranks (rank r owns
experts r*E_loc .. (r+1)*E_loc - 1), every rank routes its own tokens, sends
each kept (token, expert) row to the expert's rank, runs its experts on the
rows it received, and sends the gate-scaled outputs back for the combine
("Sparse Mixture-of-Experts (MoE): Routing Math, Load Balancing & Expert
Parallelism", section 3 dispatch / grouped GEMM / combine; "Mixture-of-Experts:
Expert Parallelism, All-to-All Routing, and Auxiliary-Loss-Free Load
Balancing", all-to-all routing).  Shared experts run on every rank's own
tokens; the bias step uses the loads summed over all ranks.

Every step on the data runs in the library's kernels (moe_route, moe_permute,
moe_gather_rows, moe_expert_ffn, moe_combine, moe_bias_update).  The exchange
is the caller's: ``DistExchange`` (torch.distributed all-to-all, NCCL on GPUs)
or ``LoopbackExchange`` (all ranks in one process, the rows moved by device
copies -- for running and testing the whole path on one GPU).  The plan of an
exchange (splits, regroup maps) is host arithmetic on the per-expert row
counts of all ranks (``plan_dispatch``).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np

from . import (MoeConfig, alloc_workspace, moe_bias_update, moe_combine, moe_expert_ffn,
               moe_expert_ffn_workspace_size, moe_gather_rows, moe_permute, moe_route,
               moe_workspace_size)


@dataclass
class Plan:
    send_splits: List[int]      # rows this rank sends to each rank (its experts' rows of x_perm)
    recv_splits: List[int]      # rows this rank receives from each rank
    regroup: np.ndarray         # target row -> received row (expert-major order)
    local_offsets: np.ndarray   # [E_loc + 1] rows of each local expert after the regroup
    n_send: int
    n_recv: int


def plan_dispatch(offsets_all: np.ndarray, rank: int, world: int) -> Plan:
    """offsets_all[src] = the [E_r + 1] expert offsets of rank src's permuted rows.
    Rows of expert e sit at offsets[e] .. offsets[e+1]; rank r owns experts
    r*E_loc .. (r+1)*E_loc - 1, so what rank src sends to rank r is one
    contiguous range of its rows.  Received rows arrive source by source
    (expert-major within a source); the regroup orders them expert by expert,
    sources ascending, each source's rows in their order."""
    offs = np.asarray(offsets_all, np.int64)
    E_r = offs.shape[1] - 1
    assert E_r % world == 0, "E_r must divide evenly over the ranks"
    E_loc = E_r // world
    cnt = np.diff(offs, axis=1)                                    # [W, E_r]
    lo, hi = rank * E_loc, (rank + 1) * E_loc
    send = [int(offs[rank, (r + 1) * E_loc] - offs[rank, r * E_loc]) for r in range(world)]
    mine = cnt[:, lo:hi]                                           # [W_src, E_loc]
    recv = [int(x) for x in mine.sum(axis=1)]
    local_offsets = np.concatenate([[0], np.cumsum(mine.sum(axis=0))]).astype(np.int32)
    src_base = np.concatenate([[0], np.cumsum(recv)])[:-1]        # first received row of each source
    regroup = np.empty(int(mine.sum()), np.int32)
    for e in range(E_loc):
        at = local_offsets[e]
        for src in range(world):
            n = int(mine[src, e])
            first = src_base[src] + int(mine[src, :e].sum())
            regroup[at:at + n] = np.arange(first, first + n)
            at += n
    return Plan(send, recv, regroup, local_offsets, int(sum(send)), int(sum(recv)))


class DistExchange:
    """All-to-all over torch.distributed (every rank calls the same methods)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)

    # the lists hold this process's single rank (the loopback form holds all ranks)
    def all_gather_offsets(self, offs):
        import torch
        out = [torch.empty_like(offs) for _ in range(self.world)]
        self.dist.all_gather(out, offs, group=self.group)
        return np.stack([o.cpu().numpy() for o in out])

    def all_to_all(self, outs, inps, out_splits, in_splits):
        (out,), (inp,), (osp,), (isp,) = outs, inps, out_splits, in_splits
        self.dist.all_to_all_single(out, inp, list(osp), list(isp), group=self.group)

    def all_reduce_sum(self, t):
        self.dist.all_reduce(t, group=self.group)


class ExpertParallelLayer:
    """One rank's share of an expert-parallel MoE layer (bf16 or fp32).

    cfg: the layer's config with T = this rank's tokens and E_r = all routed
    experts.  w_gate/w_up/w_down: this rank's E_r / W routed experts;
    ws_*: the shared experts (every rank holds them)."""

    def __init__(self, cfg: MoeConfig, rank: int, world: int, e, w_gate, w_up, w_down,
                 ws_gate=None, ws_up=None, ws_down=None, device="cuda"):
        import torch
        self.torch = torch
        self.cfg, self.rank, self.world = cfg, rank, world
        self.E_loc = cfg.E_r // world
        self.e, self.W = e, (w_gate, w_up, w_down)
        self.WS = (ws_gate, ws_up, ws_down)
        self.dt = torch.bfloat16 if cfg.dtype == 1 else torch.float32
        T, K, d = cfg.T, cfg.K, cfg.d_model
        self.ws = alloc_workspace(moe_workspace_size(cfg), device)
        max_recv = world * T * K
        self.ws_ffn = alloc_workspace(moe_expert_ffn_workspace_size(cfg, self.E_loc, cfg.d_ffn, max_recv), device)
        self.ws_sh = (alloc_workspace(moe_expert_ffn_workspace_size(cfg, 1, cfg.d_ffn_shared, T), device)
                      if cfg.E_s else None)
        i32 = dict(dtype=torch.int32, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        self.idx = torch.empty((T, K), **i32)
        self.gates = torch.empty((T, K), **f32)
        self.counts = torch.empty(cfg.E_r, **i32)
        self.offsets = torch.empty(cfg.E_r + 1, **i32)
        self.perm_tok = torch.empty(T * K, **i32)
        self.row_of = torch.empty((T, K), **i32)
        self.kept = torch.empty(cfg.E_r, **i32)
        self.row_gate = torch.empty(T * K, **f32)
        self.x_perm = torch.empty((T * K, d), dtype=self.dt, device=device)
        self.out_perm = torch.empty_like(self.x_perm)
        self.shared_out = torch.empty((max(cfg.E_s, 1), T, d), dtype=self.dt, device=device)
        self.device = device

    # phase 1: route and permute this rank's tokens (s_in: fed fp32 scores, for tests)
    def route(self, h, b, s_in=None):
        moe_route(self.cfg, h, self.e, b, s_in, None, self.idx, self.gates, self.counts, self.ws)
        moe_permute(self.cfg, self.idx, self.gates, h, self.offsets, self.perm_tok, self.row_of, self.kept,
                    self.row_gate, self.x_perm, self.ws)

    # phase 2: this rank's experts on the rows it received (x_recv, g_recv)
    def experts(self, plan: Plan, x_recv, g_recv):
        torch = self.torch
        n = plan.n_recv
        es = x_recv.element_size() * self.cfg.d_model
        out_recv = torch.empty_like(x_recv)
        if n == 0:
            return out_recv
        regroup = torch.from_numpy(plan.regroup).to(self.device)
        x_grp, g_grp = torch.empty_like(x_recv), torch.empty_like(g_recv)
        moe_gather_rows(x_recv, n, es, regroup, n, x_grp)
        moe_gather_rows(g_recv, n, 4, regroup, n, g_grp)
        out_grp = torch.empty_like(x_recv)
        moe_expert_ffn(self.cfg, self.E_loc, self.cfg.d_ffn, n, torch.from_numpy(plan.local_offsets).to(self.device),
                       x_grp, self.W[0], self.W[1], self.W[2], g_grp, out_grp, self.ws_ffn)
        inverse = np.empty_like(plan.regroup)
        inverse[plan.regroup] = np.arange(n, dtype=np.int32)
        moe_gather_rows(out_grp, n, es, torch.from_numpy(inverse).to(self.device), n, out_recv)
        return out_recv

    # phase 3: shared experts, combine
    def combine(self, h, y):
        torch = self.torch
        T = self.cfg.T
        if self.cfg.E_s:
            off = torch.tensor([0, T], dtype=torch.int32, device=self.device)
            for j in range(self.cfg.E_s):
                moe_expert_ffn(self.cfg, 1, self.cfg.d_ffn_shared, T, off, h, self.WS[0][j:j + 1],
                               self.WS[1][j:j + 1], self.WS[2][j:j + 1], None, self.shared_out[j], self.ws_sh)
        moe_combine(self.cfg, h, self.out_perm, self.shared_out if self.cfg.E_s else None, self.row_of, y)


def forward(layers: List[ExpertParallelLayer], hs, b, ys, exchange, gamma: float = 0.0,
            update_bias: bool = False, max_vio=None, s_in: Optional[list] = None):
    """One expert-parallel layer step.  With ``LoopbackExchange`` ``layers``,
    ``hs`` and ``ys`` hold every rank; with ``DistExchange`` one entry each
    (this process's rank).  ``b`` is the shared bias (updated in place with the
    loads summed over the ranks when update_bias)."""
    import torch
    for i, (L, h) in enumerate(zip(layers, hs)):
        L.route(h, b, None if s_in is None else s_in[i])
    offs_all = exchange.all_gather_offsets(*[L.offsets for L in layers])
    plans = [plan_dispatch(offs_all, L.rank, L.world) for L in layers]
    d = layers[0].cfg.d_model
    x_recv = [torch.empty((p.n_recv, d), dtype=L.dt, device=L.device) for L, p in zip(layers, plans)]
    g_recv = [torch.empty(p.n_recv, dtype=torch.float32, device=L.device) for L, p in zip(layers, plans)]
    exchange.all_to_all(x_recv, [L.x_perm[:p.n_send] for L, p in zip(layers, plans)],
                        [p.recv_splits for p in plans], [p.send_splits for p in plans])
    exchange.all_to_all(g_recv, [L.row_gate[:p.n_send] for L, p in zip(layers, plans)],
                        [p.recv_splits for p in plans], [p.send_splits for p in plans])
    out_recv = [L.experts(p, x, g) for L, p, x, g in zip(layers, plans, x_recv, g_recv)]
    exchange.all_to_all([L.out_perm[:p.n_send] for L, p in zip(layers, plans)], out_recv,
                        [p.send_splits for p in plans], [p.recv_splits for p in plans])
    for L, h, y in zip(layers, hs, ys):
        L.combine(h, y)
    if update_bias or max_vio is not None:
        total = [L.counts.clone() for L in layers]
        exchange.all_reduce_sum(*total)
        L0 = layers[0]
        cfg_g = MoeConfig.from_buffer_copy(L0.cfg)
        cfg_g.T = L0.cfg.T * L0.world                               # the loads of the whole batch
        moe_bias_update(cfg_g, total[0], gamma if update_bias else 0.0, b, max_vio)
    return plans


class LoopbackExchange:
    """All ranks in one process: the same steps as DistExchange, the rows
    moved by device copies (torch slicing) instead of a collective."""

    def __init__(self, world: int):
        self.world = world

    def all_gather_offsets(self, *offs):
        return np.stack([o.cpu().numpy() for o in offs])

    def all_to_all(self, outs, inps, out_splits, in_splits):
        W = self.world
        for dst in range(W):
            at = 0
            for src in range(W):
                first = int(sum(in_splits[src][:dst]))
                n = in_splits[src][dst]
                assert n == out_splits[dst][src]
                outs[dst][at:at + n].copy_(inps[src][first:first + n])
                at += n

    def all_reduce_sum(self, *ts):
        total = ts[0].clone()
        for t in ts[1:]:
            total += t
        for t in ts:
            t.copy_(total)

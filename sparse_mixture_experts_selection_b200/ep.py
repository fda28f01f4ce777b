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
moe_ep_plan, moe_gather_rows, moe_expert_ffn, moe_combine, moe_bias_update).
The exchange is the caller's: ``DistExchange`` (torch.distributed: NCCL on
device tensors; gloo through host copies) or ``LoopbackExchange`` (all ranks
in one process, the rows moved by device copies -- for running and testing
the whole path on one GPU).  The plan of an exchange (splits, regroup maps)
is built on the device by moe_ep_plan from the all-gathered per-expert
offsets; only the 2 x W split sizes are copied to the host, because the
all-to-all takes them there.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

from . import (MoeConfig, alloc_workspace, moe_bias_update, moe_combine, moe_ep_plan, moe_expert_ffn,
               moe_expert_ffn_workspace_size, moe_gather_rows, moe_permute, moe_route,
               moe_workspace_size)


@dataclass
class Plan:
    send_splits: List[int]      # rows this rank sends to each rank (its experts' rows of x_perm)
    recv_splits: List[int]      # rows this rank receives from each rank
    regroup: "object"           # device int32 [n_recv]: regrouped row -> received row (expert-major)
    inverse: "object"           # device int32 [n_recv]: received row -> regrouped row
    local_offsets: "object"     # device int32 [E_loc + 1]: rows of each local expert after the regroup
    n_send: int
    n_recv: int


class DistExchange:
    """All-to-all over torch.distributed (every rank calls the same methods).
    NCCL moves device tensors directly; gloo (CPU collectives) goes through
    host copies of the same tensors."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.host = dist.get_backend(group) == "gloo"

    # the lists hold this process's single rank (the loopback form holds all ranks)
    def all_gather_offsets(self, offs):
        """[W, E_r + 1] int32 on offs' device: every rank's expert offsets."""
        import torch
        src = offs.cpu() if self.host else offs
        out = [torch.empty_like(src) for _ in range(self.world)]
        self.dist.all_gather(out, src, group=self.group)
        return torch.stack(out).to(offs.device)

    def all_to_all(self, outs, inps, out_splits, in_splits):
        (out,), (inp,), (osp,), (isp,) = outs, inps, out_splits, in_splits
        if self.host:
            o = out.new_empty(out.shape, device="cpu")
            self.dist.all_to_all_single(o, inp.cpu(), list(osp), list(isp), group=self.group)
            out.copy_(o)
        else:
            self.dist.all_to_all_single(out, inp, list(osp), list(isp), group=self.group)

    def all_reduce_sum(self, t):
        if self.host:
            c = t.cpu()
            self.dist.all_reduce(c, group=self.group)
            t.copy_(c)
        else:
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
        if cfg.dtype not in (0, 1):
            raise ValueError(f"ExpertParallelLayer supports fp32 (0) and bf16 (1) layers, not dtype {cfg.dtype}")
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
        # exchange plan (moe_ep_plan): splits, local offsets, regroup and inverse maps
        self.max_recv = max_recv
        self.splits = torch.empty(2 * world, **i32)
        self.local_offsets = torch.empty(self.E_loc + 1, **i32)
        self.regroup = torch.empty(max(max_recv, 1), **i32)
        self.inverse = torch.empty(max(max_recv, 1), **i32)
        self.err = torch.zeros(1, **i32)
        self.device = device

    # the exchange plan from every rank's offsets [W, E_r + 1] (device); the
    # split sizes are the only values copied to the host
    def plan(self, offsets_all) -> Plan:
        moe_ep_plan(offsets_all, self.world, self.rank, self.cfg.E_r, self.max_recv, self.splits,
                    self.local_offsets, self.regroup, self.inverse, self.err)
        sp = self.splits.cpu().tolist()
        send, recv = sp[:self.world], sp[self.world:]
        n_recv = int(sum(recv))
        if n_recv > self.max_recv:
            raise RuntimeError(f"expert-parallel plan: {n_recv} rows would arrive, room for {self.max_recv}")
        return Plan(send, recv, self.regroup[:n_recv], self.inverse[:n_recv], self.local_offsets,
                    int(sum(send)), n_recv)

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
        x_grp, g_grp = torch.empty_like(x_recv), torch.empty_like(g_recv)
        moe_gather_rows(x_recv, n, es, plan.regroup, n, x_grp)
        moe_gather_rows(g_recv, n, 4, plan.regroup, n, g_grp)
        out_grp = torch.empty_like(x_recv)
        moe_expert_ffn(self.cfg, self.E_loc, self.cfg.d_ffn, n, plan.local_offsets,
                       x_grp, self.W[0], self.W[1], self.W[2], g_grp, out_grp, self.ws_ffn)
        moe_gather_rows(out_grp, n, es, plan.inverse, n, out_recv)
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
    plans = [L.plan(offs_all) for L in layers]
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
        import torch
        return torch.stack(offs)

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

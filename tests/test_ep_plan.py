"""Host logic of the expert-parallel exchange (no GPU): the reference plan's
splits and regroup map (the restatement the device plan moe_ep_plan is
compared with on the GPU) against a direct enumeration of the (rank, token,
expert) rows, the same plan on two gloo ranks from the gathered offsets, and
DistExchange's gloo path against the loopback exchange."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_oracle as mo
from ep_reference import plan_reference as plan_dispatch


def test_plan_hand_example():
    offs = np.array([[0, 1, 3, 6, 6], [0, 2, 2, 3, 7]])       # 2 ranks, 4 experts
    p0, p1 = plan_dispatch(offs, 0, 2), plan_dispatch(offs, 1, 2)
    assert p0.send_splits == [3, 3] and p0.recv_splits == [3, 2]
    assert list(p0.local_offsets) == [0, 3, 5] and list(p0.regroup) == [0, 3, 4, 1, 2]
    assert p1.send_splits == [2, 5] and p1.recv_splits == [3, 5]
    assert list(p1.local_offsets) == [0, 4, 8] and list(p1.regroup) == list(range(8))


@pytest.mark.parametrize("W,E,K,T,cf", [(4, 16, 4, 50, 0.0), (2, 8, 2, 33, 0.0), (8, 64, 6, 40, 0.0), (4, 16, 4, 50, 0.8)])
def test_plan_matches_enumeration(W, E, K, T, cf):
    rng = np.random.default_rng(W * 100 + E)
    disp, rows_of = [], []
    for r in range(W):
        s = mo.sigmoid_scores(rng.normal(size=(T, E)).astype(np.float32))
        idx = mo.select_experts(s, np.zeros(E, np.float32), K)
        dsp = mo.dispatch(idx, E, cf)
        disp.append(dsp)
        # (rank, token, expert) of each permuted row, in the rank's row order
        rows_of.append([(r, int(t), int(e)) for e in range(E) for t in dsp.perm_tok[dsp.offsets[e]:dsp.offsets[e + 1]]])
    offs = np.stack([d.offsets for d in disp])
    E_loc = E // W
    plans = [plan_dispatch(offs, r, W) for r in range(W)]
    for r in range(W):
        for dst in range(W):
            assert plans[r].send_splits[dst] == plans[dst].recv_splits[r]
        # what rank r receives, source by source, then regrouped
        recv = []
        for src in range(W):
            first = sum(plans[src].send_splits[:r])
            recv += rows_of[src][first:first + plans[src].send_splits[r]]
        got = [recv[i] for i in plans[r].regroup]
        want = [(src, t, e) for e in range(r * E_loc, (r + 1) * E_loc) for src in range(W)
                for (s_, t, e_) in rows_of[src] if s_ == src and e_ == e]
        assert got == want
        # local offsets delimit the local experts' rows
        for j in range(E_loc):
            seg = got[plans[r].local_offsets[j]:plans[r].local_offsets[j + 1]]
            assert all(e == r * E_loc + j for (_, _, e) in seg)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(rank)
        E, K, T = 8, 2, 30
        s = mo.sigmoid_scores(rng.normal(size=(T, E)).astype(np.float32))
        offs = torch.from_numpy(mo.dispatch(mo.select_experts(s, np.zeros(E, np.float32), K), E).offsets.astype(np.int32))
        out = [torch.empty_like(offs) for _ in range(world)]
        dist.all_gather(out, offs)
        p = plan_dispatch(np.stack([o.numpy() for o in out]), rank, world)
        splits = [torch.empty(world, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(splits, torch.tensor(p.send_splits, dtype=torch.int64))
        ok = all(int(splits[src][rank]) == p.recv_splits[src] for src in range(world))
        q.put((rank, ok, p.n_recv == len(p.regroup)))
    finally:
        dist.destroy_process_group()


def test_plan_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert res == [(0, True, True), (1, True, True)]


def _rank_rows(rank, E=8, K=2, T=30, d=4):
    """One rank's permuted rows (row value = (rank, token, expert) code) and offsets."""
    rng = np.random.default_rng(rank + 7)
    s = mo.sigmoid_scores(rng.normal(size=(T, E)).astype(np.float32))
    dsp = mo.dispatch(mo.select_experts(s, np.zeros(E, np.float32), K), E)
    n = int(dsp.offsets[-1])
    ex = np.repeat(np.arange(E), np.diff(dsp.offsets))
    code = rank * 10000 + dsp.perm_tok[:n] * 10 + ex
    rows = np.repeat(code[:, None], d, axis=1).astype(np.float32)
    return torch.from_numpy(rows), torch.from_numpy(dsp.offsets.astype(np.int32))


def _exchange_worker(rank, world, port, q):
    from sparse_mixture_experts_selection_b200.ep import DistExchange, LoopbackExchange
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rows, offs = _rank_rows(rank)
        X = DistExchange()
        offs_all = X.all_gather_offsets(offs).numpy()
        plan = plan_dispatch(offs_all, rank, world)
        out = torch.empty((plan.n_recv, rows.shape[1]))
        X.all_to_all([out], [rows], [plan.recv_splits], [plan.send_splits])
        # the loopback exchange of all ranks' rows, rebuilt from the same seeds
        allr = [_rank_rows(r) for r in range(world)]
        plans = [plan_dispatch(offs_all, r, world) for r in range(world)]
        outs = [torch.empty((p.n_recv, rows.shape[1])) for p in plans]
        LoopbackExchange(world).all_to_all(outs, [a[0] for a in allr], [p.recv_splits for p in plans],
                                           [p.send_splits for p in plans])
        t = torch.tensor([float(rank + 1)])
        X.all_reduce_sum(t)
        q.put((rank, bool(torch.equal(out, outs[rank])), float(t)))
    finally:
        dist.destroy_process_group()


def test_dist_exchange_moves_the_loopback_rows_on_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 30500 + os.getpid() % 1000
    procs = [ctx.Process(target=_exchange_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert res == [(0, True, 3.0), (1, True, 3.0)]

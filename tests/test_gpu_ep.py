"""Expert-parallel layer on one GPU with the loopback exchange (W ranks in one
process, the rows moved by device copies): every rank's output against the
oracle's layer on that rank's tokens, routing bit-exact (scores fed), and the
bias step on the loads summed over the ranks bit-exact."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as mo
import sparse_mixture_experts_selection_b200 as moe
from sparse_mixture_experts_selection_b200 import ep
from gpu_helpers import BF16_TOL, HostWeights, check_close, oracle_cfg, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


@pytest.mark.parametrize("W,E_s", [(4, 1), (2, 0)])
def test_expert_parallel_loopback_matches_oracle(W, E_s):
    w = mi.WORKLOADS["deepseek_v3"].with_(T=96, d_model=128, E_r=16, E_s=E_s, K=4, d_ffn=128,
                                          d_ffn_shared=128, n_groups=4, topk_groups=2, group_topn=2)
    HW = HostWeights(w)
    Wd = HW.device()
    e, b = mi.gen_centroids(w), mi.gen_bias(w) + np.float32(0.003) * np.arange(w.E_r, dtype=np.float32)
    E_loc = w.E_r // W
    cfg = moe.config_for(w)
    layers = [ep.ExpertParallelLayer(cfg, r, W, to_dev(e), Wd["gate"][r * E_loc:(r + 1) * E_loc],
                                     Wd["up"][r * E_loc:(r + 1) * E_loc], Wd["down"][r * E_loc:(r + 1) * E_loc],
                                     Wd["sgate"], Wd["sup"], Wd["sdown"]) for r in range(W)]
    hs = [mi.gen_h(w, step) for step in range(W)]                # each rank its own tokens
    ss = [mo.affinity(h, e, w.score_fn) for h in hs]
    bd = to_dev(b)
    ys = [torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda") for _ in range(W)]
    mv = torch.empty(1, dtype=torch.float32, device="cuda")
    ep.forward(layers, [to_dev(h, torch.bfloat16) for h in hs], bd, ys, ep.LoopbackExchange(W), gamma=0.01,
               update_bias=True, max_vio=mv, s_in=[to_dev(s) for s in ss])
    torch.cuda.synchronize()
    counts = np.zeros(w.E_r, np.int64)
    for r in range(W):
        ref = mo.layer_forward(oracle_cfg(w), hs[r], e, b, HW.source(), s_in=ss[r])
        assert np.array_equal(layers[r].idx.cpu().numpy(), ref["idx"])
        check_close(ys[r].float().cpu().numpy(), ref["y"], hs[r], BF16_TOL, True, 2.0 ** -8)
        counts += ref["counts"]
    want_b = mo.bias_update(b, counts, w.K, W * w.T, 0.01)
    assert np.array_equal(bd.cpu().numpy().view(np.int32), want_b.view(np.int32))
    assert np.float32(mv.item()) == np.float32(mo.max_vio(counts, w.K, W * w.T, w.E_r))


# ---------------------------------------------------------------------------
# the exchange plan built on the device (moe_ep_plan) against the reference
# restatement (itself pinned to an enumeration of the rows in test_ep_plan.py)
# ---------------------------------------------------------------------------

def _offsets(W, E, K, T, cf, seed, empty_rank=None):
    rng = np.random.default_rng(seed)
    out = []
    for r in range(W):
        if r == empty_rank:
            out.append(np.zeros(E + 1, np.int64))
            continue
        s = mo.sigmoid_scores(rng.normal(size=(T, E)).astype(np.float32))
        out.append(mo.dispatch(mo.select_experts(s, np.zeros(E, np.float32), K), E, cf).offsets)
    return np.stack(out).astype(np.int32)


@pytest.mark.parametrize("W,E,K,T,cf,empty", [(4, 16, 4, 50, 0.0, None), (2, 8, 2, 33, 0.0, None),
                                              (8, 64, 6, 40, 0.0, 3), (4, 16, 4, 50, 0.8, None),
                                              (1, 32, 4, 20, 0.0, None), (64, 1024, 8, 96, 0.0, None)])
def test_ep_plan_matches_reference(W, E, K, T, cf, empty):
    from ep_reference import plan_reference
    offs = _offsets(W, E, K, T, cf, W * 31 + E, empty)
    od = to_dev(offs, torch.int32)
    E_loc = E // W
    max_recv = W * T * K
    for rank in sorted({0, W - 1, W // 2}):
        ref = plan_reference(offs, rank, W)
        splits = torch.empty(2 * W, dtype=torch.int32, device="cuda")
        loc = torch.empty(E_loc + 1, dtype=torch.int32, device="cuda")
        regroup = torch.full((max_recv,), -7, dtype=torch.int32, device="cuda")
        inverse = torch.full((max_recv,), -7, dtype=torch.int32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        moe.moe_ep_plan(od, W, rank, E, max_recv, splits, loc, regroup, inverse, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        sp = splits.cpu().numpy()
        assert sp[:W].tolist() == ref.send_splits and sp[W:].tolist() == ref.recv_splits
        assert np.array_equal(loc.cpu().numpy(), ref.local_offsets)
        n = ref.n_recv
        rg = regroup.cpu().numpy()
        assert np.array_equal(rg[:n], ref.regroup) and np.all(rg[n:] == -7)
        inv = inverse.cpu().numpy()
        assert np.array_equal(inv[:n][ref.regroup], np.arange(n)) and np.all(inv[n:] == -7)


def test_ep_plan_reports_overflow_without_writing_maps():
    offs = _offsets(4, 16, 4, 50, 0.0, 5)
    from ep_reference import plan_reference
    ref = plan_reference(offs, 1, 4)
    max_recv = ref.n_recv - 1                      # one row too few
    splits = torch.empty(8, dtype=torch.int32, device="cuda")
    loc = torch.empty(5, dtype=torch.int32, device="cuda")
    regroup = torch.full((max_recv,), -7, dtype=torch.int32, device="cuda")
    inverse = torch.full((max_recv,), -7, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_ep_plan(to_dev(offs, torch.int32), 4, 1, 16, max_recv, splits, loc, regroup, inverse, err)
    torch.cuda.synchronize()
    assert int(err.item()) == moe.DEVERR_INDEX
    assert splits.cpu().numpy()[4:].sum() == ref.n_recv       # the split sizes still tell the caller
    assert np.all(regroup.cpu().numpy() == -7) and np.all(inverse.cpu().numpy() == -7)


# ---------------------------------------------------------------------------
# DistExchange end to end: two processes (one rank each) on this GPU, the
# exchange over gloo through host copies -- nothing on the GPU waits on the
# other rank; every rank's output against the oracle on its tokens
# ---------------------------------------------------------------------------

def _ep_workload():
    return mi.WORKLOADS["deepseek_v3"].with_(T=80, d_model=128, E_r=16, E_s=1, K=4, d_ffn=128,
                                             d_ffn_shared=128, n_groups=4, topk_groups=2, group_topn=2)


def _dist_worker(rank, world, port, q):
    import os
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        w = _ep_workload()
        HW = HostWeights(w)
        Wd = HW.device()
        e = mi.gen_centroids(w)
        b = mi.gen_bias(w) + np.float32(0.003) * np.arange(w.E_r, dtype=np.float32)
        E_loc = w.E_r // world
        L = ep.ExpertParallelLayer(moe.config_for(w), rank, world, to_dev(e),
                                   Wd["gate"][rank * E_loc:(rank + 1) * E_loc],
                                   Wd["up"][rank * E_loc:(rank + 1) * E_loc],
                                   Wd["down"][rank * E_loc:(rank + 1) * E_loc], Wd["sgate"], Wd["sup"], Wd["sdown"])
        h = mi.gen_h(w, rank)
        s = mo.affinity(h, e, w.score_fn)
        bd = to_dev(b)
        y = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
        mv = torch.empty(1, dtype=torch.float32, device="cuda")
        ep.forward([L], [to_dev(h, torch.bfloat16)], bd, [y], ep.DistExchange(), gamma=0.01, update_bias=True,
                   max_vio=mv, s_in=[to_dev(s)])
        torch.cuda.synchronize()
        ref = mo.layer_forward(oracle_cfg(w), h, e, b, HW.source(), s_in=s)
        ok_idx = bool(np.array_equal(L.idx.cpu().numpy(), ref["idx"]))
        try:
            check_close(y.float().cpu().numpy(), ref["y"], h, BF16_TOL, True, 2.0 ** -8)
            ok_y = True
        except AssertionError as ex:
            ok_y = repr(ex)
        q.put((rank, ok_idx, ok_y, bd.cpu().numpy().tolist(), float(mv.item()), ref["counts"].tolist()))
    except Exception as ex:          # reported to the parent, which fails the test
        q.put((rank, "error", repr(ex), None, None, None))
    finally:
        dist.destroy_process_group()


def test_dist_exchange_two_ranks_gloo_end_to_end():
    import os
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 31500 + os.getpid() % 1000
    procs = [ctx.Process(target=_dist_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=120)
    for r in res:
        assert r[1] is True and r[2] is True, r
    w = _ep_workload()
    b = mi.gen_bias(w) + np.float32(0.003) * np.arange(w.E_r, dtype=np.float32)
    counts = np.array(res[0][5]) + np.array(res[1][5])
    want_b = mo.bias_update(b, counts, w.K, 2 * w.T, 0.01)
    for r in res:                      # both ranks hold the same bias, stepped on the summed loads
        assert np.array_equal(np.array(r[3], np.float32).view(np.int32), want_b.view(np.int32))
        assert np.float32(r[4]) == np.float32(mo.max_vio(counts, w.K, 2 * w.T, w.E_r))

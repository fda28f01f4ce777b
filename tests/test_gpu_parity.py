"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on small
seeded workloads that span several tiles and ragged tails.

Routing, counts, permutation and bias are compared bit for bit when the GPU is
fed the oracle's fp32 scores; with its own fp32 logits the GPU must agree on
every token whose K-th / (K+1)-th key gap (and group-score gap) is >= 1e-5.
Layer outputs must satisfy max|y - y_ref| <= 2e-2 * RMS (bf16) or 1e-4 * RMS
(fp32), against both RMS(y_ref) and RMS(y_ref - h).
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from moe_inputs import native
from oracle import moe_oracle as mo
import sparse_mixture_experts_selection_b200 as moe
from gpu_helpers import (BF16_TOL, F32_TOL, HostWeights, Layer, check_close, oracle_cfg, out_eps_of,
                         to_dev, torch_dtype)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

W = mi.WORKLOADS
# small versions of every workload: several 128-row tiles per expert, ragged
# row/column/K tails, shared experts, groups, capacity
SMALL = {
    "toy_fp32": W["toy_fp32"].with_(steps=1),
    "mixtral_small": W["mixtral_8x14336"].with_(T=300, d_model=256, d_ffn=320),
    "finegrained_small": W["finegrained_64x1408"].with_(T=600, d_model=192, E_r=16, E_s=2, K=4,
                                                        d_ffn=192, d_ffn_shared=136),
    "finegrained_small_cf": W["finegrained_64x1408_cf1.25"].with_(T=600, d_model=192, E_r=16, E_s=2,
                                                                  K=4, d_ffn=192, d_ffn_shared=136),
    # ~110 rows per expert: full, partial (97..127 rows) and transposed short
    # (<= 96 rows) tiles side by side
    "finegrained_near_tile": W["finegrained_64x1408"].with_(T=440, d_model=192, E_r=16, E_s=2, K=4,
                                                           d_ffn=192, d_ffn_shared=136),
    "deepseek_small": W["deepseek_v3"].with_(T=520, d_model=256, E_r=64, E_s=1, K=6, d_ffn=256,
                                             d_ffn_shared=384, n_groups=8, topk_groups=3),
    "decode_small": W["deepseek_v3_decode"].with_(T=24, d_model=320, E_r=64, d_ffn=128,
                                                  d_ffn_shared=128, topk_groups=4),
    # >= 512 rows per routed expert: the GEMMs run on CTA pairs (256-row tiles)
    "mixtral_pairs": W["mixtral_8x14336"].with_(T=2304, d_model=256, d_ffn=320),
    "finegrained_pairs": W["finegrained_64x1408"].with_(T=1100, d_model=192, E_r=8, E_s=2, K=4,
                                                        d_ffn=192, d_ffn_shared=136),
    # T = 4 * 256 + 40: the shared experts' last 40 rows ride as merged tails
    "finegrained_pairs_shared_tail": W["finegrained_64x1408"].with_(T=1064, d_model=192, E_r=8, E_s=2,
                                                                    K=4, d_ffn=192, d_ffn_shared=136),
}


def tol_of(w):
    return BF16_TOL if w.dtype != "f32" else F32_TOL


def inputs(w, step=0):
    h = mi.gen_h(w, step)
    e = mi.gen_centroids(w)
    b = mi.gen_bias(w)
    return h, e, b


# ---------------------------------------------------------------------------
# input generator twin on the device
# ---------------------------------------------------------------------------

def test_device_generator_matches_numpy():
    for bf16 in (False, True):
        for tid, start, n, sigma in [(4, 0, 5000, 0.02), (9, 3 * 2**30 + 11, 777, 1.0)]:
            t = torch.empty(n, dtype=torch.bfloat16 if bf16 else torch.float32, device="cuda")
            native.fill_device(t.data_ptr(), n, bf16, 1003, tid, start, sigma)
            ref = mi.normal_f32(1003, tid, start, n, sigma)
            got = t.view(torch.int16 if bf16 else torch.int32).cpu().numpy()
            want = mi.f32_to_bf16_bits(ref).view(np.int16) if bf16 else ref.view(np.int32)
            assert np.array_equal(got, want)


# ---------------------------------------------------------------------------
# routing (a1-a4)
# ---------------------------------------------------------------------------

def _route_gpu(cfg, s_in=None, h=None, e=None, b=None):
    T, K, E = cfg.T, cfg.K, cfg.E_r
    ws = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    gates = torch.empty((T, K), dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    s_out = torch.empty((T, E), dtype=torch.float32, device="cuda")
    moe.moe_route(cfg, h, e, b, s_in, s_out, idx, gates, counts, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    return idx.cpu().numpy(), gates.cpu().numpy(), counts.cpu().numpy(), s_out.cpu().numpy()


ROUTE_CASES = [
    # (T, E, K, n_groups, topk_groups, group_topn, score_fn, coarse)
    (1000, 64, 8, 1, 1, 0, 0, False),
    (777, 256, 8, 8, 4, 2, 0, False),
    (513, 8, 2, 1, 1, 0, 1, False),
    (300, 6, 6, 1, 1, 0, 0, False),        # K = E_r
    (400, 64, 8, 1, 1, 0, 0, True),        # many exact ties
    (400, 256, 8, 8, 4, 2, 0, True),       # ties inside the group logic too
    (333, 1024, 16, 32, 8, 3, 0, False),   # widest supported shape
    (129, 16, 3, 4, 2, 1, 0, True),
]


@pytest.mark.parametrize("case", ROUTE_CASES, ids=[str(c) for c in ROUTE_CASES])
def test_route_fed_scores_bit_exact(case):
    T, E, K, ng, tg, gn, fn, coarse = case
    rng = np.random.default_rng(T * 7 + E)
    if coarse:
        s = (rng.integers(0, 16, size=(T, E)) / 16).astype(np.float32)
        b = (rng.integers(-2, 3, size=E) / 64).astype(np.float32)
    else:
        z = rng.normal(size=(T, E)).astype(np.float32)
        s = mo.sigmoid_scores(z) if fn == 0 else mo.softmax_scores(z)
        b = rng.uniform(-0.02, 0.02, size=E).astype(np.float32)
    if fn == 1:
        b = np.zeros(E, np.float32)
    cfg = moe.MoeConfig(T=T, d_model=64, E_r=E, E_s=0, K=K, d_ffn=64, d_ffn_shared=0, score_fn=fn,
                        n_groups=ng, topk_groups=tg, group_topn=gn, capacity_factor=0.0, dtype=0,
                        add_residual=1)
    idx, gates, counts, s_out = _route_gpu(cfg, s_in=to_dev(s), b=to_dev(b))
    want_idx = mo.select_experts(s, b, K, ng, tg, gn)
    want_g = mo.gates_from_scores(s, want_idx)
    assert np.array_equal(s_out.view(np.int32), s.view(np.int32))
    assert np.array_equal(idx, want_idx)
    assert np.array_equal(gates.view(np.int32), want_g.view(np.int32))
    assert np.array_equal(counts, mo.load_counts(want_idx, E))


@pytest.mark.parametrize("name", ["toy_fp32", "mixtral_small", "deepseek_small", "decode_small"])
def test_route_independent_logits(name):
    w = SMALL[name]
    h, e, b = inputs(w)
    cfg = moe.config_for(w)
    b_sel = b if w.score_fn == 0 else np.zeros(w.E_r, np.float32)
    idx, gates, counts, s_gpu = _route_gpu(cfg, h=to_dev(h, torch_dtype(w)), e=to_dev(e), b=to_dev(b))
    s_ref = mo.affinity(h, e, w.score_fn)
    # fp32 logits vs the double-evaluated ones: a few ulp of the logit
    assert np.max(np.abs(s_gpu.astype(np.float64) - s_ref)) < 2e-6
    want = mo.select_experts(s_ref, b_sel, w.K, w.n_groups, w.topk_groups, w.group_topn)
    fragile = mo.near_tie_tokens(s_ref, b_sel, w.K, w.n_groups, w.topk_groups, w.group_topn, 1e-5)
    bad = np.any(idx != want, axis=1) & ~fragile
    assert not bad.any(), np.nonzero(bad)[0][:10]
    assert fragile.mean() < 0.05


# ---------------------------------------------------------------------------
# dispatch (a5)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("cf", [0.0, 1.25, 0.5, 100.0])
def test_permute_bit_exact(cf):
    T, E, K, d = 1100, 32, 4, 64
    rng = np.random.default_rng(5)
    s = mo.sigmoid_scores(rng.normal(size=(T, E)).astype(np.float32) + np.linspace(0, 2, E, dtype=np.float32))
    idx = mo.select_experts(s, np.zeros(E, np.float32), K)
    gates = mo.gates_from_scores(s, idx)
    h = rng.normal(size=(T, d)).astype(np.float32)
    cfg = moe.MoeConfig(T=T, d_model=d, E_r=E, E_s=0, K=K, d_ffn=64, d_ffn_shared=0, score_fn=0,
                        n_groups=1, topk_groups=1, group_topn=0, capacity_factor=cf, dtype=0,
                        add_residual=1)
    ws = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    dev = dict(offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"),
               perm_tok=torch.full((T * K,), -7, dtype=torch.int32, device="cuda"),
               row_of=torch.empty((T, K), dtype=torch.int32, device="cuda"),
               kept=torch.empty(E, dtype=torch.int32, device="cuda"),
               row_gate=torch.empty(T * K, dtype=torch.float32, device="cuda"),
               x_perm=torch.zeros((T * K, d), dtype=torch.float32, device="cuda"))
    hd = to_dev(h)
    moe.moe_permute(cfg, to_dev(idx.astype(np.int32), torch.int32), to_dev(gates), hd, dev["offsets"],
                    dev["perm_tok"], dev["row_of"], dev["kept"], dev["row_gate"], dev["x_perm"], ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    ref = mo.dispatch(idx, E, cf)
    n = int(ref.offsets[-1])
    assert np.array_equal(dev["offsets"].cpu().numpy(), ref.offsets)
    assert np.array_equal(dev["kept"].cpu().numpy(), ref.kept)
    assert np.array_equal(dev["perm_tok"].cpu().numpy()[:n], ref.perm_tok)
    assert np.array_equal(dev["row_of"].cpu().numpy(), ref.row_of)
    rg = dev["row_gate"].cpu().numpy()[:n]
    assert np.array_equal(rg.view(np.int32), gates[ref.perm_tok, ref.perm_slot].view(np.int32))
    assert np.array_equal(dev["x_perm"].cpu().numpy()[:n], h[ref.perm_tok])


@pytest.mark.parametrize("dtype,d", [("f32", 8192), ("bf16", 4104), ("f32", 8)])
def test_permute_row_gather_widths(dtype, d):
    """x_perm = h[perm_tok] bit for bit across row widths: 32 KB fp32 rows leave
    room for only three row buffers in the bulk-copy ring, so the row gather
    falls back to its per-lane copy; 8208-byte bf16 rows take the ring with
    an odd number of 16-byte chunks; 32-byte rows the ring's smallest rows;
    rows past the kept ones stay untouched."""
    T, E, K = 300, 16, 3
    rng = np.random.default_rng(11)
    s = mo.sigmoid_scores(rng.normal(size=(T, E)).astype(np.float32))
    idx = mo.select_experts(s, np.zeros(E, np.float32), K)
    h = rng.normal(size=(T, d)).astype(np.float32)
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    if dtype == "bf16":
        h = mi.round_bf16(h)
    cfg = moe.MoeConfig(T=T, d_model=d, E_r=E, E_s=0, K=K, d_ffn=64, d_ffn_shared=0, score_fn=0,
                        n_groups=1, topk_groups=1, group_topn=0, capacity_factor=1.0,
                        dtype=0 if dtype == "f32" else 1, add_residual=1)
    ws = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    z = lambda *sh: torch.empty(sh, dtype=torch.int32, device="cuda")
    x_perm = torch.full((T * K, d), 3.0, dtype=dt, device="cuda")
    offsets, perm_tok = z(E + 1), z(T * K)
    moe.moe_permute(cfg, to_dev(idx.astype(np.int32), torch.int32), None, to_dev(h, dt), offsets, perm_tok,
                    z(T, K), z(E), None, x_perm, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    ref = mo.dispatch(idx, E, 1.0)
    n = int(ref.offsets[-1])
    assert n < T * K                                  # capacity 1.0 drops some pairs
    got = x_perm.float().cpu().numpy()
    assert np.array_equal(got[:n], h[ref.perm_tok])
    assert np.all(got[n:] == 3.0)


def test_permute_rejects_bad_expert_index():
    """An out-of-range expert index sets the device error word (no fault)."""
    T, E, K = 64, 8, 2
    idx = np.tile(np.array([[0, 9]], np.int32), (T, 1))
    cfg = moe.MoeConfig(T=T, d_model=64, E_r=E, E_s=0, K=K, d_ffn=64, d_ffn_shared=0, score_fn=0,
                        n_groups=1, topk_groups=1, group_topn=0, capacity_factor=0.0, dtype=0,
                        add_residual=1)
    ws = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    z = lambda *s: torch.zeros(s, dtype=torch.int32, device="cuda")
    moe.moe_permute(cfg, to_dev(idx, torch.int32), None, None, z(E + 1), z(T * K), z(T, K), z(E),
                    None, None, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == moe.DEVERR_INDEX
    moe.moe_clear_device_error(ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0


# ---------------------------------------------------------------------------
# experts (a6-a7), combine (a8), bias (a9)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,d", [("bf16", 192), ("bf16", 200), ("f32", 192)])
def test_expert_ffn_entry(dtype, d):
    """Rows 130 and 257 end in merged tails, the 1-row expert is a transposed
    tile; d = 200 leaves the down GEMM's last 32-column block of a warp
    partly past the output width (the staged epilogue's element-wise edge)."""
    n_exp, f = 5, 200
    rows = np.array([0, 130, 0, 257, 1], dtype=np.int64)     # empty groups and ragged tiles
    offsets = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    R = int(offsets[-1])
    rng = np.random.default_rng(3)
    rnd = lambda *s, sc=1.0: (rng.normal(size=s) * sc).astype(np.float32)
    x, wg, wu = rnd(R, d), rnd(n_exp, f, d, sc=d ** -0.5), rnd(n_exp, f, d, sc=d ** -0.5)
    wd, scale = rnd(n_exp, d, f, sc=f ** -0.5), rng.uniform(0.1, 1, size=R).astype(np.float32)
    if dtype == "bf16":
        x, wg, wu, wd = (mi.round_bf16(a) for a in (x, wg, wu, wd))
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    cfg = moe.MoeConfig(T=R, d_model=d, E_r=n_exp, E_s=0, K=1, d_ffn=f, d_ffn_shared=0, score_fn=0,
                        n_groups=1, topk_groups=1, group_topn=0, capacity_factor=0.0,
                        dtype=1 if dtype == "bf16" else 0, add_residual=1)
    max_rows = R + 3
    assert moe.moe_expert_ffn_tile_rows(cfg, n_exp, max_rows) == (128 if dtype == "bf16" else 32)
    ws = moe.alloc_workspace(moe.moe_expert_ffn_workspace_size(cfg, n_exp, f, max_rows))
    xd = torch.zeros((max_rows, d), dtype=dt, device="cuda")
    xd[:R] = to_dev(x, dt)
    out = torch.full((max_rows, d), 7.0, dtype=dt, device="cuda")
    moe.moe_expert_ffn(cfg, n_exp, f, max_rows, to_dev(offsets, torch.int32), xd, to_dev(wg, dt),
                       to_dev(wu, dt), to_dev(wd, dt), to_dev(scale), out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    got = out.float().cpu().numpy()
    want = np.zeros((R, d))
    for g in range(n_exp):
        a, b_ = offsets[g], offsets[g + 1]
        if b_ > a:
            want[a:b_] = scale[a:b_, None] * mo.swiglu(x[a:b_], wg[g], wu[g], wd[g])
    # the act and the output are stored in bf16 (fp32): allow the output's own
    # rounding (2^-8 |want|, twice the unit roundoff) on top of the tolerance
    eps = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -22
    tol = BF16_TOL if dtype == "bf16" else F32_TOL
    err = np.max(np.abs(got[:R] - want) - eps * np.abs(want))
    assert err <= tol * np.sqrt(np.mean(want ** 2)), err
    assert np.all(got[R:] == 7.0)                     # rows past offsets[n] untouched


# Rows per expert reaching every CTA-pair tile kind (256-row tiles; the even
# CTA holds rows 0..127 of a tile, the odd one rows 128..255): empty, one row,
# a full even half with the odd half empty, one row in the odd half, one full
# tile, merged tails of 1, 44 and 64 rows (the largest) after one tile and of
# 48 rows after two, a tile + 65 rows (the smallest padded tail) and + 127
# (even half partial, odd empty), two tiles + 188 rows (odd half partial).
PAIR_ROWS = [0, 1, 128, 129, 256, 257, 300, 320, 560, 321, 383, 700]


def test_expert_ffn_pair_tiles():
    """moe_expert_ffn with >= 512 rows provisioned per expert (the CTA-pair
    GEMMs), ragged gate/up and down column tiles (f = 200, d = 192): every
    output row within the bar, rows past offsets[n] untouched."""
    n_exp, d, f = len(PAIR_ROWS), 192, 200
    rows = np.array(PAIR_ROWS, dtype=np.int64)
    offsets = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    R = int(offsets[-1])
    rng = np.random.default_rng(5)
    rnd = lambda *s, sc=1.0: (rng.normal(size=s) * sc).astype(np.float32)
    x = mi.round_bf16(rnd(R, d))
    wg, wu = mi.round_bf16(rnd(n_exp, f, d, sc=d ** -0.5)), mi.round_bf16(rnd(n_exp, f, d, sc=d ** -0.5))
    wd = mi.round_bf16(rnd(n_exp, d, f, sc=f ** -0.5))
    scale = rng.uniform(0.1, 1, size=R).astype(np.float32)
    cfg = moe.MoeConfig(T=R, d_model=d, E_r=n_exp, E_s=0, K=1, d_ffn=f, d_ffn_shared=0, score_fn=0,
                        n_groups=1, topk_groups=1, group_topn=0, capacity_factor=0.0, dtype=1, add_residual=1)
    max_rows = 512 * n_exp
    assert moe.moe_expert_ffn_tile_rows(cfg, n_exp, max_rows) == 256        # CTA pairs
    ws = moe.alloc_workspace(moe.moe_expert_ffn_workspace_size(cfg, n_exp, f, max_rows))
    xd = torch.zeros((max_rows, d), dtype=torch.bfloat16, device="cuda")
    xd[:R] = to_dev(x, torch.bfloat16)
    out = torch.full((max_rows, d), 7.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(cfg, n_exp, f, max_rows, to_dev(offsets, torch.int32), xd, to_dev(wg, torch.bfloat16),
                       to_dev(wu, torch.bfloat16), to_dev(wd, torch.bfloat16), to_dev(scale), out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    got = out.float().cpu().numpy()
    for g in range(n_exp):
        a, b_ = offsets[g], offsets[g + 1]
        if b_ == a:
            continue
        want = scale[a:b_, None] * mo.swiglu(x[a:b_], wg[g], wu[g], wd[g])
        err = np.max(np.abs(got[a:b_] - want) - 2.0 ** -8 * np.abs(want))
        assert err <= BF16_TOL * np.sqrt(np.mean(want ** 2)), (g, PAIR_ROWS[g], err)
    assert np.all(got[R:] == 7.0)                     # rows past offsets[n] untouched


def test_expert_ffn_pair_tiles_all_empty():
    """The CTA-pair GEMMs with no unit at all (every expert empty): the
    launches end cleanly, no output row is touched, no error is set."""
    n_exp, d, f = 4, 192, 200
    cfg = moe.MoeConfig(T=64, d_model=d, E_r=n_exp, E_s=0, K=1, d_ffn=f, d_ffn_shared=0, score_fn=0,
                        n_groups=1, topk_groups=1, group_topn=0, capacity_factor=0.0, dtype=1, add_residual=1)
    max_rows = 512 * n_exp
    assert moe.moe_expert_ffn_tile_rows(cfg, n_exp, max_rows) == 256
    ws = moe.alloc_workspace(moe.moe_expert_ffn_workspace_size(cfg, n_exp, f, max_rows))
    w = torch.zeros((n_exp, f, d), dtype=torch.bfloat16, device="cuda")
    wd = torch.zeros((n_exp, d, f), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((max_rows, d), dtype=torch.bfloat16, device="cuda")
    out = torch.full((max_rows, d), 7.0, dtype=torch.bfloat16, device="cuda")
    offsets = torch.zeros(n_exp + 1, dtype=torch.int32, device="cuda")
    moe.moe_expert_ffn(cfg, n_exp, f, max_rows, offsets, x, w, w, wd, None, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    assert bool((out.float() == 7.0).all())


@pytest.mark.parametrize("dtype,K", [("bf16", 3), ("f32", 3), ("bf16", 8), ("bf16", 2)])
def test_combine_entry_fixed_order(dtype, K):
    T, d, E_s, R = 77, 64, 2, 200
    rng = np.random.default_rng(4)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    h = rng.normal(size=(T, d)).astype(np.float32)
    slot = rng.normal(size=(R, d)).astype(np.float32)
    shared = rng.normal(size=(E_s, T, d)).astype(np.float32)
    if dtype == "bf16":
        h, slot, shared = (mi.round_bf16(a) for a in (h, slot, shared))
    row_of = rng.integers(-1, R, size=(T, K)).astype(np.int32)
    cfg = moe.MoeConfig(T=T, d_model=d, E_r=8, E_s=E_s, K=K, d_ffn=64, d_ffn_shared=64, score_fn=0,
                        n_groups=1, topk_groups=1, group_topn=0, capacity_factor=0.0,
                        dtype=1 if dtype == "bf16" else 0, add_residual=1)
    y = torch.empty((T, d), dtype=dt, device="cuda")
    moe.moe_combine(cfg, to_dev(h, dt), to_dev(slot, dt), to_dev(shared, dt), to_dev(row_of, torch.int32), y)
    torch.cuda.synchronize()
    # fixed order in fp32: h, shared j = 0.., slots k = 0.. (kept only); one rounding
    acc = h.copy()
    for j in range(E_s):
        acc = (acc + shared[j]).astype(np.float32)
    for k in range(K):
        m = row_of[:, k] >= 0
        add = np.where(m[:, None], slot[np.maximum(row_of[:, k], 0)], np.float32(0))
        acc = np.where(m[:, None], (acc + add).astype(np.float32), acc)
    want = mi.round_bf16(acc) if dtype == "bf16" else acc
    assert np.array_equal(y.float().cpu().numpy().view(np.int32), want.view(np.int32))


def test_bias_update_entry_bit_exact():
    E, K, T = 64, 8, 1000
    rng = np.random.default_rng(6)
    counts = rng.multinomial(K * T, np.ones(E) / E).astype(np.int32)
    counts[3] = K * T // E                                  # exactly the fair share: no step
    b = rng.uniform(-0.01, 0.01, size=E).astype(np.float32)
    cfg = moe.MoeConfig(T=T, d_model=64, E_r=E, E_s=0, K=K, d_ffn=64, d_ffn_shared=0, score_fn=0,
                        n_groups=1, topk_groups=1, group_topn=0, capacity_factor=0.0, dtype=0,
                        add_residual=1)
    bd, mv = to_dev(b), torch.empty(1, dtype=torch.float32, device="cuda")
    moe.moe_bias_update(cfg, to_dev(counts, torch.int32), 0.001, bd, mv)
    torch.cuda.synchronize()
    want = mo.bias_update(b, counts.astype(np.int64), K, T, 0.001)
    assert np.array_equal(bd.cpu().numpy().view(np.int32), want.view(np.int32))
    assert mv.item() == np.float32(mo.max_vio(counts.astype(np.int64), K, T, E))


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", sorted(SMALL))
def test_layer_gemm_tile_choice(name):
    """bf16 layers provisioning >= 512 rows per routed expert (T*K/E_r) take
    the CTA-pair GEMMs, the others the single-CTA ones; fp32 the CUDA cores."""
    w = SMALL[name]
    want = 32 if w.dtype == "f32" else (256 if w.T * w.K >= 512 * w.E_r else 128)
    assert moe.moe_expert_ffn_tile_rows(moe.config_for(w), w.E_r, w.T * w.K) == want
    if "_pairs" in name:
        assert want == 256


@pytest.mark.parametrize("name", sorted(SMALL))
def test_layer_fed_scores(name):
    """Layer with the oracle's fp32 scores fed in: routing, counts and kept rows
    bit-exact; y within tolerance on every token."""
    w = SMALL[name]
    h, e, b = inputs(w)
    HW = HostWeights(w)
    cfg = oracle_cfg(w)
    s = mo.affinity(h, e, w.score_fn)
    ref = mo.layer_forward(cfg, h, e, b, HW.source(), s_in=s)
    L = Layer(w, HW.device())
    y = L.forward(to_dev(h, torch_dtype(w)), None, to_dev(b), s_in=to_dev(s))
    assert L.device_error() == 0
    assert np.array_equal(L.idx.cpu().numpy(), ref["idx"])
    assert np.array_equal(L.gates.cpu().numpy().view(np.int32), ref["gates"].view(np.int32))
    assert np.array_equal(L.counts.cpu().numpy(), ref["counts"])
    assert np.array_equal(L.kept.cpu().numpy(), ref["kept"])
    assert np.float32(L.max_vio.item()) == np.float32(ref["max_vio"])
    check_close(y.float().cpu().numpy(), ref["y"], h, tol_of(w), bool(w.add_residual), out_eps_of(w))


@pytest.mark.parametrize("name", sorted(SMALL))
def test_layer_independent(name):
    """Layer computing its own fp32 logits: every non-fragile token routes as
    the oracle does and its output is within tolerance."""
    w = SMALL[name]
    h, e, b = inputs(w)
    HW = HostWeights(w)
    ref = mo.layer_forward(oracle_cfg(w), h, e, b, HW.source())
    L = Layer(w, HW.device())
    y = L.forward(to_dev(h, torch_dtype(w)), to_dev(e), to_dev(b)).float().cpu().numpy()
    assert L.device_error() == 0
    b_sel = b if w.score_fn == 0 else np.zeros(w.E_r, np.float32)
    fragile = mo.near_tie_tokens(ref["s"], b_sel, w.K, w.n_groups, w.topk_groups, w.group_topn, 1e-5)
    same = np.all(L.idx.cpu().numpy() == ref["idx"], axis=1)
    assert np.all(same | fragile)
    if w.capacity_factor > 0 and not np.all(same):
        pytest.skip("a fragile token moved a capacity boundary")
    ok = same
    check_close(y[ok], ref["y"][ok], h[ok], tol_of(w), bool(w.add_residual), out_eps_of(w))


@pytest.mark.parametrize("name", ["mixtral_small", "finegrained_pairs"])
def test_layer_slot_saturation_reports_range(name):
    """The layer keeps its slot and shared rows in fp16: down weights scaled by
    2^20 (exact in bf16) push them past 65504; they saturate, the output stays
    finite and the device error word reads MOE_DEVERR_RANGE -- on the
    single-CTA and on the CTA-pair GEMMs.  The unscaled layer reports nothing."""
    w = SMALL[name]
    h, e, b = inputs(w)
    HW = HostWeights(w)
    Wd = HW.device()
    L = Layer(w, Wd)
    L.forward(to_dev(h, torch_dtype(w)), to_dev(e), to_dev(b))
    assert L.device_error() == 0
    Wd["down"].mul_(2.0 ** 20)
    if Wd["sdown"] is not None:
        Wd["sdown"].mul_(2.0 ** 20)
    y = L.forward(to_dev(h, torch_dtype(w)), to_dev(e), to_dev(b))
    assert L.device_error() == moe.DEVERR_RANGE
    assert torch.isfinite(y.float()).all()
    assert float(y.float().abs().max()) > 65504.0 / 2


def test_layer_deterministic_and_workspace_reuse():
    w = SMALL["deepseek_small"]
    h, e, b = inputs(w)
    HW = HostWeights(w)
    L = Layer(w, HW.device())
    hd, ed, bd = to_dev(h, torch_dtype(w)), to_dev(e), to_dev(b)
    y1 = L.forward(hd, ed, bd).clone()
    y2 = L.forward(hd, ed, bd).clone()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_toy_bias_chain_60_steps():
    """The toy aux-loss-free run: 60 steps of fresh tokens with gamma = 0.1.
    Per step the GPU is fed the oracle's scores; idx, counts, MaxVio and the
    carried bias are bit-exact at every step and y is within 1e-4 * RMS."""
    w = W["toy_fp32"]
    e = mi.gen_centroids(w)
    HW = HostWeights(w)
    cfg = oracle_cfg(w)
    L = Layer(w, HW.device())
    b_ref = mi.gen_bias(w)
    bd = to_dev(b_ref)
    vio = []
    for step in range(w.steps):
        h = mi.gen_h(w, step)
        s = mo.affinity(h, e, w.score_fn)
        ref = mo.layer_forward(cfg, h, e, b_ref, HW.source(), s_in=s)
        y = L.forward(to_dev(h), None, bd, s_in=to_dev(s), update_bias=True, gamma=w.gamma)
        assert np.array_equal(L.idx.cpu().numpy(), ref["idx"]), step
        assert np.array_equal(L.counts.cpu().numpy(), ref["counts"]), step
        b_ref = mo.bias_update(b_ref, ref["counts"], w.K, w.T, w.gamma)
        assert np.array_equal(bd.cpu().numpy().view(np.int32), b_ref.view(np.int32)), step
        assert np.float32(L.max_vio.item()) == np.float32(ref["max_vio"])
        check_close(y.cpu().numpy(), ref["y"], h, F32_TOL, True, 2.0 ** -22)
        vio.append(ref["max_vio"])
    assert L.device_error() == 0
    print("toy MaxVio per step:", np.round(vio, 3).tolist())


EDGE = {
    "single_token": SMALL["deepseek_small"].with_(T=1),
    "dense_E1_K1": SMALL["finegrained_small"].with_(E_r=1, K=1),
    "all_dropped": SMALL["finegrained_small_cf"].with_(capacity_factor=0.001),
    "K_equals_E_softmax": SMALL["mixtral_small"].with_(K=8),
    "hot_expert_3_row_tiles": SMALL["deepseek_small"].with_(T=700, centroid_skew="zipf_1.2"),
    "E1024_groups32": W["deepseek_v3"].with_(T=200, d_model=64, E_r=1024, E_s=1, K=16, d_ffn=64,
                                             d_ffn_shared=64, n_groups=32, topk_groups=8, group_topn=3),
    "no_residual": SMALL["finegrained_small"].with_(add_residual=0),
}


@pytest.mark.parametrize("name", sorted(EDGE))
def test_layer_edge_cases(name):
    w = EDGE[name]
    h, e, b = inputs(w)
    HW = HostWeights(w)
    s = mo.affinity(h, e, w.score_fn)
    ref = mo.layer_forward(oracle_cfg(w), h, e, b, HW.source(), s_in=s)
    L = Layer(w, HW.device())
    y = L.forward(to_dev(h, torch_dtype(w)), None, to_dev(b), s_in=to_dev(s))
    assert L.device_error() == 0
    assert np.array_equal(L.idx.cpu().numpy(), ref["idx"])
    assert np.array_equal(L.kept.cpu().numpy(), ref["kept"])
    if name == "all_dropped":
        assert ref["kept"].sum() == 0
    if name == "hot_expert_3_row_tiles":
        assert ref["kept"].max() > 2 * 128
    check_close(y.float().cpu().numpy(), ref["y"], h, tol_of(w), bool(w.add_residual), out_eps_of(w))


def test_bounded_wait_reports_timeout_without_fault():
    """A pipeline wait that can never complete gives up after its limit, sets
    MOE_DEVERR_WAIT_TIMEOUT in the workspace's error word and returns; the
    context stays usable (a layer call afterwards still matches the oracle)."""
    ws = moe.alloc_workspace(4096)
    moe.moe_selftest_bounded_wait(ws, 20_000_000)          # 20 ms
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == moe.DEVERR_WAIT_TIMEOUT
    moe.moe_clear_device_error(ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    test_route_fed_scores_bit_exact(ROUTE_CASES[0])

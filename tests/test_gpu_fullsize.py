"""Full-size workloads in the launch configuration bench.py times.

Routing is checked on every token (fed with the oracle's fp32 scores: bit-exact;
with the GPU's own logits: identical outside the 1e-5 near-tie set, which must
stay below 1 % of the tokens).  Layer outputs are checked on a stratified
sample of at least 32 tokens chosen so that every tile kind of the grouped
GEMMs that the routing produces is reached (see row_kinds), for which the
oracle evaluates the experts in float64 from weights regenerated on the host
by the generator's C twin (the device copy comes from its CUDA twin; both equal
the numpy definition bit for bit).  Tile kinds the real routing does not
produce at a given shape are reached on purpose by the expert-FFN entry point
with constructed row counts at the same d and f, compared row by row.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as mo
import sparse_mixture_experts_selection_b200 as moe
from gpu_helpers import (BF16_TOL, Layer, LazyHostWeights, check_close, device_weights, oracle_cfg,
                         out_eps_of, to_dev, torch_dtype)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

FULL = ["mixtral_8x14336", "finegrained_64x1408", "finegrained_64x1408_cf1.25", "deepseek_v3",
        "deepseek_v3_decode"]
N_SAMPLE = 32          # tokens per stratified sample (at most T)
PER_KIND = 4           # rows sampled per tile kind

# Tile geometry of the grouped GEMMs under test: 128-row tiles; a last tile of
# at most 64 rows rides in the unit of the full tile before it ("merged_tail",
# computed transposed, and "full_with_tail" for that full tile); any other
# tile of at most 96 rows runs transposed ("transposed"); 97-127 rows run as a
# padded 128-row tile ("padded"); "full" is a plain 128-row tile.
BM, MERGE_MAX, SWAP_MAX = 128, 64, 96
KINDS = ("full", "full_with_tail", "merged_tail", "transposed", "padded")

# the kinds the seeded routing of each workload produces (checked, and each
# one must be reached by the sample)
EXPECTED_KINDS = {
    "mixtral_8x14336": {"full", "full_with_tail", "merged_tail", "transposed"},
    "finegrained_64x1408": set(KINDS),
    "finegrained_64x1408_cf1.25": set(KINDS),
    "deepseek_v3": set(KINDS),
    "deepseek_v3_decode": {"transposed"},
}


def row_kinds(offsets):
    """Tile kind of every permuted row, from the per-expert row offsets."""
    offsets = np.asarray(offsets, np.int64)
    kind = np.empty(int(offsets[-1]), dtype=object)
    for ex in range(len(offsets) - 1):
        r0, n = int(offsets[ex]), int(offsets[ex + 1] - offsets[ex])
        if n == 0:
            continue
        mt = (n + BM - 1) // BM
        last = n - (mt - 1) * BM
        merged = mt >= 2 and last <= MERGE_MAX
        for t in range(mt):
            rv = min(BM, n - t * BM)
            if merged and t == mt - 1:
                k = "merged_tail"
            elif merged and t == mt - 2:
                k = "full_with_tail"
            elif rv == BM:
                k = "full"
            elif rv <= SWAP_MAX:
                k = "transposed"
            else:
                k = "padded"
            kind[r0 + t * BM:r0 + t * BM + rv] = k
    return kind


def stratified_tokens(w, disp, avoid=None, seed=7):
    """At least N_SAMPLE tokens (or all T): for every tile kind present, the
    tokens of PER_KIND of its rows in different experts -- including the last
    row of a merged tail and the first and last row of an expert -- plus
    seeded random tokens.  Returns (tokens, kinds reached)."""
    rng = np.random.default_rng(seed)
    kinds = row_kinds(disp.offsets)
    ex_of_row = np.repeat(np.arange(len(disp.offsets) - 1), np.diff(disp.offsets))
    rows = []
    reached = set()
    for k in KINDS:
        cand = np.nonzero(kinds == k)[0]
        if not len(cand):
            continue
        reached.add(k)
        picked = []
        if k == "merged_tail":
            last_rows = [r for r in cand if r + 1 == len(kinds) or ex_of_row[r + 1] != ex_of_row[r]]
            picked.append(int(last_rows[0]))
        for r in rng.permutation(cand):
            if len(picked) >= PER_KIND:
                break
            if all(ex_of_row[r] != ex_of_row[q] for q in picked):
                picked.append(int(r))
        rows += picked
    nz = np.nonzero(np.diff(disp.offsets) > 0)[0]
    if len(nz):
        ex = int(rng.choice(nz))
        rows += [int(disp.offsets[ex]), int(disp.offsets[ex + 1] - 1)]      # expert boundary rows
    tok = set(int(disp.perm_tok[r]) for r in rows)
    pool = np.arange(w.T) if avoid is None else np.nonzero(~avoid)[0]
    for t in rng.permutation(pool):
        if len(tok) >= min(N_SAMPLE, w.T):
            break
        tok.add(int(t))
    return np.array(sorted(tok)), reached


@pytest.fixture(scope="module")
def weights_cache():
    return {}


def _layer(w, cache):
    if w.name.split("_cf")[0] not in cache:
        cache.clear()
        torch.cuda.empty_cache()
        cache[w.name.split("_cf")[0]] = device_weights(w)
    return Layer(w, cache[w.name.split("_cf")[0]])


@pytest.mark.parametrize("name", FULL)
def test_fullsize_fed_routing_and_sampled_outputs(name, weights_cache):
    w = mi.WORKLOADS[name]
    h, e, b = mi.gen_h(w), mi.gen_centroids(w), mi.gen_bias(w)
    cfg = oracle_cfg(w)
    s = mo.affinity(h, e, w.score_fn)
    b_sel = b if w.score_fn == 0 else np.zeros(w.E_r, np.float32)
    idx, gates, disp = mo.route(cfg, s, b_sel)
    L = _layer(w, weights_cache)
    y = L.forward(to_dev(h, torch_dtype(w)), None, to_dev(b), s_in=to_dev(s))
    assert L.device_error() == 0
    assert np.array_equal(L.idx.cpu().numpy(), idx)
    assert np.array_equal(L.gates.cpu().numpy().view(np.int32), gates.view(np.int32))
    assert np.array_equal(L.counts.cpu().numpy(), disp.counts)
    assert np.array_equal(L.kept.cpu().numpy(), disp.kept)
    tok, reached = stratified_tokens(w, disp)
    assert reached == EXPECTED_KINDS[name], (sorted(reached), sorted(EXPECTED_KINDS[name]))
    # a token with a dropped pair must still be sampled when one exists
    if w.capacity_factor > 0:
        dropped = np.nonzero((disp.row_of < 0).any(axis=1))[0]
        if len(dropped):
            tok = np.unique(np.concatenate([tok, dropped[:1]]))
    assert len(tok) >= min(N_SAMPLE, w.T)
    y_ref = mo.layer_output(cfg, h, idx, gates, disp, LazyHostWeights(w).source(), tokens=tok)
    check_close(y.float().cpu().numpy()[tok], y_ref, h[tok], BF16_TOL, True, out_eps_of(w))
    print(f"{name}: {len(tok)} tokens checked, tile kinds reached: {sorted(reached)}")


@pytest.mark.parametrize("name", FULL)
def test_fullsize_independent_routing(name, weights_cache):
    w = mi.WORKLOADS[name]
    h, e, b = mi.gen_h(w), mi.gen_centroids(w), mi.gen_bias(w)
    s = mo.affinity(h, e, w.score_fn)
    b_sel = b if w.score_fn == 0 else np.zeros(w.E_r, np.float32)
    want = mo.select_experts(s, b_sel, w.K, w.n_groups, w.topk_groups, w.group_topn)
    fragile = mo.near_tie_tokens(s, b_sel, w.K, w.n_groups, w.topk_groups, w.group_topn, 1e-5)
    L = _layer(w, weights_cache)
    L.forward(to_dev(h, torch_dtype(w)), to_dev(e), to_dev(b))
    assert L.device_error() == 0
    s_gpu = L.s.cpu().numpy()
    assert np.max(np.abs(s_gpu.astype(np.float64) - s)) < 5e-6
    got = L.idx.cpu().numpy()
    bad = np.any(got != want, axis=1) & ~fragile
    assert not bad.any(), (np.nonzero(bad)[0][:10], fragile.sum())
    # the exemption must stay rare: 1 % of the tokens, at least 4 (measured with
    # the seeded inputs: Mixtral 1 of 4096, fine-grained 8 of 8192, DeepSeek-V3
    # 14 of 4096, decode 2 of 64)
    assert int(fragile.sum()) <= max(4, w.T // 100), int(fragile.sum())
    print(f"{name}: {int(fragile.sum())} of {w.T} tokens within 1e-5 of a tie")


def test_deepseek_bias_chain_20_steps(weights_cache):
    """DeepSeek-V3 shape, 20 steps of fresh tokens with gamma = 0.001: routing,
    counts, MaxVio and the carried bias bit-exact at every step (GPU fed with
    the oracle's scores); sampled outputs checked at the first and last step."""
    w = mi.WORKLOADS["deepseek_v3"]
    e = mi.gen_centroids(w)
    b_ref = mi.gen_bias(w)
    cfg = oracle_cfg(w)
    L = _layer(w, weights_cache)
    bd = to_dev(b_ref)
    src = LazyHostWeights(w).source()
    for step in range(w.steps):
        h = mi.gen_h(w, step)
        s = mo.affinity(h, e, 0)
        idx, gates, disp = mo.route(cfg, s, b_ref)
        y = L.forward(to_dev(h, torch.bfloat16), None, bd, s_in=to_dev(s), update_bias=True, gamma=w.gamma)
        assert np.array_equal(L.idx.cpu().numpy(), idx), step
        assert np.array_equal(L.counts.cpu().numpy(), disp.counts), step
        assert np.float32(L.max_vio.item()) == np.float32(mo.max_vio(disp.counts, w.K, w.T, w.E_r)), step
        b_ref = mo.bias_update(b_ref, disp.counts, w.K, w.T, w.gamma)
        assert np.array_equal(bd.cpu().numpy().view(np.int32), b_ref.view(np.int32)), step
        if step in (0, w.steps - 1):
            tok, _ = stratified_tokens(w, disp, seed=step)
            y_ref = mo.layer_output(cfg, h, idx, gates, disp, src, tokens=tok)
            check_close(y.float().cpu().numpy()[tok], y_ref, h[tok], BF16_TOL, True, 2.0 ** -8)
    assert L.device_error() == 0


# constructed row counts reaching every tile kind: two full tiles + a 40-row
# merged tail, a 64-row tile (transposed), 96 (transposed, the largest), 97 and
# 127 (padded), a full tile + an 80-row tile (transposed, standalone), an
# empty expert, and a full tile + a 64-row merged tail (the largest merged)
CONSTRUCTED_ROWS = [296, 64, 96, 97, 127, 208, 0, 192]


@pytest.mark.parametrize("name", ["mixtral_8x14336", "finegrained_64x1408", "deepseek_v3"])
def test_fullsize_every_tile_kind(name, weights_cache):
    """moe_expert_ffn at the workload's full d and f (the Mixtral reduction is
    4096 deep, DeepSeek-V3's 7168 = 112 k-blocks), with row counts that reach
    every tile kind; every output row of every expert is compared element by
    element with g * SwiGLU(x) of the oracle (float64)."""
    w = mi.WORKLOADS[name]
    n = min(len(CONSTRUCTED_ROWS), w.E_r)
    rows = np.array(CONSTRUCTED_ROWS[:n])
    offsets = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    R = int(offsets[-1])
    kinds = row_kinds(offsets)
    assert set(kinds) == set(KINDS), sorted(set(kinds))
    x = mi.gen_h(w, 0)[np.arange(R) % w.T]
    gate = np.random.default_rng(3).uniform(0.05, 1.0, size=R).astype(np.float32)
    Wd = _layer(w, weights_cache).W
    cfg = moe.config_for(w)
    assert moe.moe_expert_ffn_tile_rows(cfg, n, R) == BM                  # the single-CTA tiles
    ws = moe.alloc_workspace(moe.moe_expert_ffn_workspace_size(cfg, n, w.d_ffn, R))
    out = torch.empty((R, w.d_model), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(cfg, n, w.d_ffn, R, to_dev(offsets, torch.int32), to_dev(x, torch.bfloat16),
                       Wd["gate"][:n], Wd["up"][:n], Wd["down"][:n], to_dev(gate), out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    got = out.float().cpu().numpy().astype(np.float64)
    src = LazyHostWeights(w).source()
    for ex in range(n):
        r0, r1 = int(offsets[ex]), int(offsets[ex + 1])
        if r0 == r1:
            continue
        want = gate[r0:r1, None].astype(np.float64) * mo.swiglu(x[r0:r1], src("gate", ex), src("up", ex),
                                                                   src("down", ex))
        diff = np.abs(got[r0:r1] - want) - 2.0 ** -8 * np.abs(want)
        r = float(np.sqrt(np.mean(want ** 2)))
        assert float(diff.max()) <= BF16_TOL * r, (ex, sorted(set(kinds[r0:r1])), float(diff.max()), r)
    print(f"{name}: every row of {n} experts ({R} rows) within the bar; kinds {sorted(set(kinds))}")


# rows per expert reaching every CTA-pair tile kind (256-row tiles: the even
# CTA holds rows 0..127, the odd one 128..255): two tiles + 188 rows (odd half
# partial), one row, one row in the odd half, merged tails of 64 rows (the
# largest) and of 48 rows after two tiles, a tile + 65 rows (the smallest
# padded tail), a tile + 1 row (merged), an empty expert
PAIR_ROWS = [700, 1, 129, 320, 560, 321, 257, 0]


@pytest.mark.parametrize("name", ["mixtral_8x14336", "finegrained_64x1408"])
def test_fullsize_pair_tiles(name, weights_cache):
    """moe_expert_ffn on the CTA-pair GEMMs (>= 512 rows provisioned per
    expert, as the layer provisions T*K/E_r at these shapes) at the workload's
    full d and f; every output row of every expert element by element."""
    w = mi.WORKLOADS[name]
    n = min(len(PAIR_ROWS), w.E_r)
    rows = np.array(PAIR_ROWS[:n])
    offsets = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    R = int(offsets[-1])
    max_rows = 512 * n
    assert moe.moe_expert_ffn_tile_rows(moe.config_for(w), n, max_rows) == 256     # CTA pairs
    x = mi.gen_h(w, 0)[np.arange(R) % w.T]
    gate = np.random.default_rng(4).uniform(0.05, 1.0, size=R).astype(np.float32)
    Wd = _layer(w, weights_cache).W
    cfg = moe.config_for(w)
    ws = moe.alloc_workspace(moe.moe_expert_ffn_workspace_size(cfg, n, w.d_ffn, max_rows))
    xd = torch.zeros((max_rows, w.d_model), dtype=torch.bfloat16, device="cuda")
    xd[:R] = to_dev(x, torch.bfloat16)
    out = torch.empty((max_rows, w.d_model), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(cfg, n, w.d_ffn, max_rows, to_dev(offsets, torch.int32), xd,
                       Wd["gate"][:n], Wd["up"][:n], Wd["down"][:n], to_dev(gate), out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    got = out[:R].float().cpu().numpy().astype(np.float64)
    src = LazyHostWeights(w).source()
    for ex in range(n):
        r0, r1 = int(offsets[ex]), int(offsets[ex + 1])
        if r0 == r1:
            continue
        want = gate[r0:r1, None].astype(np.float64) * mo.swiglu(x[r0:r1], src("gate", ex), src("up", ex),
                                                                   src("down", ex))
        diff = np.abs(got[r0:r1] - want) - 2.0 ** -8 * np.abs(want)
        r = float(np.sqrt(np.mean(want ** 2)))
        assert float(diff.max()) <= BF16_TOL * r, (ex, int(rows[ex]), float(diff.max()), r)


def test_fullsize_shared_expert_slices(weights_cache):
    """The DeepSeek-V3 shared expert (all 4096 tokens, 32 full tiles at
    d = 7168) through moe_expert_ffn: the first, a middle and the last 128-row
    slice, element by element."""
    w = mi.WORKLOADS["deepseek_v3"]
    Wd = _layer(w, weights_cache).W
    h = mi.gen_h(w, 0)
    cfg = moe.config_for(w)
    offsets = np.array([0, w.T], np.int32)
    ws = moe.alloc_workspace(moe.moe_expert_ffn_workspace_size(cfg, 1, w.d_ffn_shared, w.T))
    out = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(cfg, 1, w.d_ffn_shared, w.T, to_dev(offsets, torch.int32), to_dev(h, torch.bfloat16),
                       Wd["sgate"], Wd["sup"], Wd["sdown"], None, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    got = out.float().cpu().numpy().astype(np.float64)
    src = LazyHostWeights(w).source()
    for r0 in (0, 17 * BM, w.T - BM):
        want = mo.swiglu(h[r0:r0 + BM], src("sgate", 0), src("sup", 0), src("sdown", 0))
        diff = np.abs(got[r0:r0 + BM] - want) - 2.0 ** -8 * np.abs(want)
        assert float(diff.max()) <= BF16_TOL * float(np.sqrt(np.mean(want ** 2))), r0

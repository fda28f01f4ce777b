"""Pins of the CPU oracle to what the pages and the mathematics fix.

Each pin checks the oracle against something other than itself: values the
pages print (tests/golden), brute-force enumeration, closed forms, and
reductions to library routines (torch.nn.functional in float64).  The planted
mistake tests at the end show that a plausible slip in the oracle fails at
least one pin.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import moe_oracle as mo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# pin helpers (each returns None or raises AssertionError); the planted-mistake
# tests call them after patching the oracle
# ---------------------------------------------------------------------------

def pin_worked_bias_example():
    g = _load("worked_bias_example.json")
    s = np.array(g["scores"], dtype=F32)
    E, K, T = g["E"], g["K"], s.shape[0]
    b = np.zeros(E, F32)
    for step in ("step1", "step2"):
        want = g[step]
        idx = mo.select_experts(s, b, K)
        assert idx[:, 0].tolist() == want["idx"], (step, idx[:, 0])
        c = mo.load_counts(idx, E)
        assert c.tolist() == want["counts"], (step, c)
        assert mo.max_vio(c, K, T, E) == pytest.approx(want["max_vio"], abs=0)
        b = mo.bias_update(b, c, K, T, g["gamma"])
        assert np.array_equal(b, np.array(want["bias_after"], dtype=F32)), (step, b)
        gates = mo.gates_from_scores(s, idx)
        assert np.all(gates == F32(1.0))            # K = 1: every gate is s/s = 1


def _beats(key, i, j):
    return key[i] > key[j] or (key[i] == key[j] and i < j)


def _brute_topk(key, K, eligible):
    cands = [i for i in range(len(key)) if eligible[i]]
    winners = []
    for sub in itertools.combinations(cands, K):
        rest = [j for j in cands if j not in sub]
        if all(_beats(key, i, j) for i in sub for j in rest):
            winners.append(sub)
    assert len(winners) == 1
    return list(winners[0])


def _brute_groups(key, n_groups, topk_groups, topn):
    gs = len(key) // n_groups
    G = []
    for g in range(n_groups):
        vals = sorted(key[g * gs:(g + 1) * gs], reverse=True)[:topn]
        acc = F32(vals[0])
        for v in vals[1:]:
            acc = F32(acc + F32(v))
        G.append(acc)
    winners = []
    for sub in itertools.combinations(range(n_groups), topk_groups):
        rest = [j for j in range(n_groups) if j not in sub]
        if all(_beats(G, i, j) for i in sub for j in rest):
            winners.append(sub)
    assert len(winners) == 1
    keep = set(winners[0])
    return [(i // gs) in keep for i in range(len(key))]


def pin_bruteforce_topk(seed=0, trials=60):
    rng = np.random.default_rng(seed)
    for trial in range(trials):
        E, K = [(8, 2), (16, 2), (6, 3), (5, 5), (7, 1)][trial % 5]
        # coarse values so exact ties are frequent; negative biases allowed
        s = (rng.integers(0, 6, size=(1, E)) / 8).astype(F32)
        b = (rng.integers(-3, 3, size=E) / 8).astype(F32)
        key = [float(v) for v in mo.selection_keys(s, b)[0]]
        want = sorted(_brute_topk(key, K, [True] * E))
        got = mo.select_experts(s, b, K)[0].tolist()
        assert got == want, (E, K, key, got, want)


def pin_bruteforce_grouped(seed=1, trials=60):
    rng = np.random.default_rng(seed)
    for trial in range(trials):
        n_groups, gsz, keep, K, topn = [(4, 4, 2, 3, 2), (4, 4, 1, 2, 1), (8, 2, 3, 4, 2)][trial % 3]
        E = n_groups * gsz
        s = (rng.integers(0, 5, size=(1, E)) / 8).astype(F32)
        b = (rng.integers(-4, 2, size=E) / 8).astype(F32)    # keys may be negative
        key = [float(v) for v in mo.selection_keys(s, b)[0]]
        elig = _brute_groups(key, n_groups, keep, topn)
        want = sorted(_brute_topk(key, K, elig))
        got = mo.select_experts(s, b, K, n_groups, keep, topn)[0].tolist()
        assert got == want, (key, got, want)


def pin_gates_properties(seed=2):
    rng = np.random.default_rng(seed)
    T, E, K = 300, 64, 8
    s = mo.sigmoid_scores(rng.normal(size=(T, E)).astype(F32))
    b = (rng.uniform(-0.01, 0.01, size=E)).astype(F32)
    idx = mo.select_experts(s, b, K)
    g = mo.gates_from_scores(s, idx)
    assert np.all(np.abs(g.astype(np.float64).sum(1) - 1.0) <= K * 2.0 ** -23)
    # the gate is the unbiased s renormalised over I_t (double reference)
    sel = np.take_along_axis(s, idx.astype(np.int64), 1).astype(np.float64)
    assert np.allclose(g, sel / sel.sum(1, keepdims=True), rtol=4 * 2.0 ** -24, atol=0)
    # a bias change that leaves I_t unchanged leaves the gates bit-identical
    b2 = (b + F32(1e-3) * rng.choice([-1, 1], size=E).astype(F32)).astype(F32)
    idx2 = mo.select_experts(s, b2, K)
    same = np.all(idx2 == idx, axis=1)
    assert same.sum() > T // 4
    g2 = mo.gates_from_scores(s, idx2)
    assert np.array_equal(g2[same].view(np.uint32), g[same].view(np.uint32))


def pin_counts_and_bias(seed=3):
    rng = np.random.default_rng(seed)
    T, E, K, gamma = 257, 16, 4, 0.01
    s = mo.sigmoid_scores(rng.normal(size=(T, E)).astype(F32))
    b = rng.uniform(-0.05, 0.05, size=E).astype(F32)
    idx = mo.select_experts(s, b, K)
    c = mo.load_counts(idx, E)
    assert c.sum() == K * T
    assert all(len(set(r)) == K for r in idx.tolist())
    b1 = mo.bias_update(b, c, K, T, gamma)
    step = (b1.astype(np.float64) - b.astype(np.float64))
    # every bias moves by (the fp32 rounding of) +gamma, -gamma or 0, against the load
    cbar = K * T / E
    for i in range(E):
        want = 0.0 if c[i] == cbar else (gamma if c[i] < cbar else -gamma)
        assert abs(step[i] - want) <= 2.0 ** -20 * (1 + abs(b[i])), (i, c[i], step[i])
    assert np.array_equal(mo.bias_update(b, c, K, T, 0.0), b)     # gamma = 0 freezes b


def pin_softmax_closed_form(seed=4):
    rng = np.random.default_rng(seed)
    T, E = 500, 8
    z = (rng.normal(size=(T, E)) * 2).astype(F32)
    p = mo.softmax_scores(z)
    idx = mo.select_experts(p, np.zeros(E, F32), 2)
    g = mo.gates_from_scores(p, idx)
    za = np.take_along_axis(z, idx.astype(np.int64), 1).astype(np.float64)
    # renormalised top-2 softmax = softmax over the two selected logits
    want0 = 1.0 / (1.0 + np.exp(za[:, 1] - za[:, 0]))
    ulp = np.spacing(np.abs(want0).astype(F32)).astype(np.float64)
    assert np.all(np.abs(g[:, 0] - want0) <= 4 * ulp)
    # the two selected logits are the two largest
    assert np.all(np.sort(z, 1)[:, -2:].min(1) <= za.min(1))


def pin_k_equals_e(seed=5):
    rng = np.random.default_rng(seed)
    s = mo.sigmoid_scores(rng.normal(size=(50, 6)).astype(F32))
    idx = mo.select_experts(s, np.zeros(6, F32), 6)
    assert np.array_equal(idx, np.tile(np.arange(6), (50, 1)))
    g = mo.gates_from_scores(s, idx)
    want = s.astype(np.float64) / s.astype(np.float64).sum(1, keepdims=True)
    assert np.allclose(g, want, rtol=8 * 2.0 ** -24, atol=0)


def _torch_swiglu(x, wg, wu, wd):
    x, wg, wu, wd = (torch.from_numpy(np.asarray(a, np.float64)) for a in (x, wg, wu, wd))
    return F.linear(F.silu(F.linear(x, wg)) * F.linear(x, wu), wd).numpy()


def pin_dense_reduction(seed=6):
    """E_r = K = 1: the layer is h + SwiGLU(h) + shared SwiGLU(h), a dense FFN."""
    rng = np.random.default_rng(seed)
    T, d, f, fs = 9, 12, 20, 7
    h = rng.normal(size=(T, d))
    wg, wu = rng.normal(size=(1, f, d)), rng.normal(size=(1, f, d))
    wd = rng.normal(size=(1, d, f))
    sg, su, sd = rng.normal(size=(1, fs, d)), rng.normal(size=(1, fs, d)), rng.normal(size=(1, d, fs))
    e = rng.normal(size=(1, d)).astype(F32)
    cfg = mo.LayerConfig(T=T, d_model=d, E_r=1, E_s=1, K=1)
    out = mo.layer_forward(cfg, h, e, np.zeros(1, F32), mo.array_weights(wg, wu, wd, sg, su, sd))
    want = h + _torch_swiglu(h, wg[0], wu[0], wd[0]) + _torch_swiglu(h, sg[0], su[0], sd[0])
    assert np.allclose(out["y"], want, rtol=1e-12, atol=1e-12)


def _dense_layer(h, gates_dense, W, sW, residual=1.0):
    """The layer equation summed over ALL experts with a dense gate matrix
    (zero outside I_t), using torch.nn.functional."""
    y = residual * h
    for j in range(len(sW[0])):
        y = y + _torch_swiglu(h, sW[0][j], sW[1][j], sW[2][j])
    for i in range(gates_dense.shape[1]):
        y = y + gates_dense[:, i:i + 1] * _torch_swiglu(h, W[0][i], W[1][i], W[2][i])
    return y


def pin_dense_all_experts(seed=7):
    rng = np.random.default_rng(seed)
    T, d, f, fs, E, K, Es = 40, 16, 24, 10, 6, 2, 2
    h = rng.normal(size=(T, d)).astype(F32)
    e = (rng.normal(size=(E, d)) * 0.3).astype(F32)
    b = rng.uniform(-0.05, 0.05, size=E).astype(F32)
    W = [rng.normal(size=(E, f, d)), rng.normal(size=(E, f, d)), rng.normal(size=(E, d, f))]
    sW = [rng.normal(size=(Es, fs, d)), rng.normal(size=(Es, fs, d)), rng.normal(size=(Es, d, fs))]
    cfg = mo.LayerConfig(T=T, d_model=d, E_r=E, E_s=Es, K=K)
    out = mo.layer_forward(cfg, h, e, b, mo.array_weights(*W, *sW))
    G = np.zeros((T, E))
    np.put_along_axis(G, out["idx"].astype(np.int64), out["gates"].astype(np.float64), 1)
    want = _dense_layer(h.astype(np.float64), G, W, sW)
    assert np.allclose(out["y"], want, rtol=1e-11, atol=1e-11)
    # the affinity is sigma(h . e) (library sigmoid on a float64 matmul)
    z = torch.from_numpy(h.astype(np.float64)) @ torch.from_numpy(e.astype(np.float64)).T
    assert np.allclose(out["s"], torch.sigmoid(z).numpy(), rtol=2 ** -23, atol=2 ** -24)


def pin_capacity(seed=8):
    # floor, not ceil: T*K*CF/E_r = 10*2*1.1/4 = 5.5 -> 5
    assert mo.capacity(10, 2, 4, 1.1) == 5
    assert mo.capacity(8192, 8, 64, 1.25) == 1280
    # expert 0 is chosen by all 10 tokens: the 5 lowest token indices are kept
    idx = np.array([[0, 1 + (t % 3)] for t in range(10)], dtype=np.int32)
    dsp = mo.dispatch(idx, 4, 1.1)
    assert dsp.kept.tolist() == [5, 4, 3, 3]
    assert dsp.perm_tok[:5].tolist() == [0, 1, 2, 3, 4]
    assert (dsp.row_of[5:, 0] == -1).all() and (dsp.row_of[:5, 0] >= 0).all()
    assert dsp.counts.tolist() == [10, 4, 3, 3]            # counts are pre-drop
    # CF >= E_r/K: nothing is dropped, identical to dropless
    rng = np.random.default_rng(seed)
    s = mo.sigmoid_scores(rng.normal(size=(64, 8)).astype(F32))
    idx = mo.select_experts(s, np.zeros(8, F32), 2)
    a, b = mo.dispatch(idx, 8, 4.0), mo.dispatch(idx, 8, 0.0)
    assert np.array_equal(a.row_of, b.row_of) and np.array_equal(a.perm_tok, b.perm_tok)
    # rows are grouped by expert ascending, tokens ascending inside each expert
    for ex in range(8):
        seg = b.perm_tok[b.offsets[ex]:b.offsets[ex + 1]]
        assert np.all(np.diff(seg) > 0)
        assert all(ex in idx[t] for t in seg)


def pin_permutation_properties(seed=9):
    """Routing is permutation-equivariant; capacity deliberately is not."""
    rng = np.random.default_rng(seed)
    T, E, K = 48, 8, 2
    s = mo.sigmoid_scores(rng.normal(size=(T, E)).astype(F32))
    b = rng.uniform(-0.02, 0.02, size=E).astype(F32)
    perm = rng.permutation(T)
    idx, idx_p = mo.select_experts(s, b, K), mo.select_experts(s[perm], b, K)
    assert np.array_equal(idx[perm], idx_p)
    assert np.array_equal(mo.gates_from_scores(s, idx)[perm], mo.gates_from_scores(s[perm], idx_p))
    assert np.array_equal(mo.load_counts(idx, E), mo.load_counts(idx_p, E))
    # capacity: reversing the token order changes which (token, expert) pairs drop
    idx_c = np.array([[0, 1], [0, 2], [0, 3], [1, 2]], dtype=np.int32)
    fwd = mo.dispatch(idx_c, 4, 1.0)             # C = floor(4*2*1/4) = 2
    rev = mo.dispatch(idx_c[::-1].copy(), 4, 1.0)
    kept_fwd = {(t, int(idx_c[t, k])) for t in range(4) for k in range(2) if fwd.row_of[t, k] >= 0}
    kept_rev = {(3 - t, int(idx_c[3 - t, k])) for t in range(4) for k in range(2) if rev.row_of[t, k] >= 0}
    assert kept_fwd != kept_rev
    assert (0, 0) in kept_fwd and (0, 0) not in kept_rev


def _brute_gaps(key, K, n_groups=1, topk_groups=1, topn=0):
    """Both gaps of one token by enumeration: the kept groups are the one
    subset whose every member beats every non-member; the selected experts
    likewise among the eligible ones.  Returns (top-K gap, group gap): the
    smallest selected key minus the largest eligible unselected key, and the
    smallest kept group score minus the largest dropped one (inf when there is
    nothing to compare)."""
    E = len(key)
    gs = E // n_groups
    group_gap = math.inf
    if n_groups > 1 and topn > 0:
        elig = _brute_groups(key, n_groups, topk_groups, topn)
        G = []
        for g in range(n_groups):
            vals = sorted(key[g * gs:(g + 1) * gs], reverse=True)[:topn]
            acc = F32(vals[0])
            for v in vals[1:]:
                acc = F32(acc + F32(v))
            G.append(float(acc))
        kept_g = {i // gs for i in range(E) if elig[i]}
        dropped_g = [G[g] for g in range(n_groups) if g not in kept_g]
        if dropped_g:
            group_gap = min(G[g] for g in kept_g) - max(dropped_g)
    else:
        elig = [True] * E
    sel = _brute_topk(key, K, elig)
    rest = [key[j] for j in range(E) if elig[j] and j not in sel]
    topk_gap = min(key[i] for i in sel) - max(rest) if rest else math.inf
    return topk_gap, group_gap


def pin_near_tie_bruteforce(seed=10, trials=240):
    """near_tie_tokens against enumeration.  Keys are multiples of 2^-12 (sums
    and differences exact in fp32 and float64) with a threshold of 3 * 2^-12,
    so gaps of 0 (exact ties), 1 and 2 units are fragile and 3 or more are not;
    negative keys come from negative biases."""
    rng = np.random.default_rng(seed)
    unit = 2.0 ** -12
    thr = 3 * unit
    shapes = [(1, 8, 1, 2, 0), (1, 6, 1, 3, 0), (1, 5, 1, 4, 0), (4, 4, 2, 3, 2), (4, 4, 1, 2, 1),
              (8, 2, 3, 4, 2), (4, 2, 2, 4, 2), (4, 4, 3, 5, 2)]
    seen = set()
    for trial in range(trials):
        n_groups, gsz, keep, K, topn = shapes[trial % len(shapes)]
        E = n_groups * gsz
        T = 6
        s = (rng.integers(0, 24, size=(T, E)) * unit).astype(F32)
        b = (rng.integers(-12, 4, size=E) * unit).astype(F32)
        keys = mo.selection_keys(s, b)
        got = mo.near_tie_tokens(s, b, K, n_groups, keep, topn, gap=thr)
        for t in range(T):
            key = [float(v) for v in keys[t]]
            tg, gg = _brute_gaps(key, K, n_groups, keep, topn)
            want = tg < thr or gg < thr
            assert bool(got[t]) == want, (n_groups, gsz, keep, K, topn, key, tg, gg, bool(got[t]))
            seen.add((want, tg < thr, gg < thr))
    # both kinds of fragility, and robust tokens, all occurred
    assert {(True, True, False), (True, False, True), (False, False, False)} <= seen, seen


def pin_near_tie_handbuilt():
    """Hand-built tokens with known gaps.  Threshold 2^-17 with gaps of 2^-18
    (fragile), exactly 2^-17 (not: the rule is strict) and 2^-16 (not), and the
    default 1e-5 with gaps of about 0.5e-5 (fragile) and 2e-5 (not)."""
    def one(key, K, gap, n_groups=1, keep=1, topn=0, b=None):
        key = np.asarray(key, np.float64)
        bb = np.zeros(len(key), F32) if b is None else np.asarray(b, F32)
        s = (key - bb.astype(np.float64)).astype(F32)[None, :]
        assert np.array_equal(mo.selection_keys(s, bb)[0].astype(np.float64), key), "keys not exact"
        return bool(mo.near_tie_tokens(s, bb, K, n_groups, keep, topn, gap=gap)[0])

    u = 2.0 ** -17
    base = [0.75, 0.5, 0.25, 0.125, 0.0625, 0.03125, 0.015625, 0.0078125]
    for delta, want in ((u / 2, True), (u, False), (2 * u, False)):
        k = list(base)
        k[2] = k[1] - delta                      # K = 2: 2nd vs 3rd largest
        assert one(k, 2, u) == want, delta
        kn = [v - 1.0 for v in k]                # the same gaps on negative keys (negative bias)
        assert one(kn, 2, u, b=[-1.0] * 8) == want, delta
    k = list(base)
    k[1] = k[0] - u / 2                          # a tie inside the selected set is harmless
    assert one(k, 2, u) is False
    k = list(base)
    k[3] = k[2] - u / 2                          # a tie among the unselected ones is harmless
    assert one(k, 2, u) is False
    # default threshold 1e-5 (fp32 keys near 0.5: spacing 6e-8)
    for delta, want in ((0.5e-5, True), (2e-5, False)):
        k = [float(F32(v)) for v in (0.9, 0.5, 0.5 - delta, 0.1)]
        assert one(k, 2, 1e-5) == want, delta

    # 4 groups of 4, keep 2, group score = top-2 sum, K = 2; keys listed group by group
    def g4(*groups):
        return [v for grp in groups for v in (list(grp) + [0.0] * (4 - len(grp)))]
    # group scores 1.0, 0.5, 0.5 - delta, 0.0625: fragile exactly when delta < threshold
    for delta, want in ((u / 2, True), (u, False), (2 * u, False)):
        k = g4((0.5, 0.5), (0.25, 0.25), (0.25, 0.25 - delta), (0.0625,))
        assert one(k, 2, u, 4, 2, 2) == want, delta
    # the two DROPPED groups tie (0.25 and 0.25), kept groups far apart: harmless;
    # the best groups are not in index order (scores 1.0, 0.25, 0.25, 0.5)
    assert one(g4((0.5, 0.5), (0.125, 0.125), (0.125, 0.125), (0.25, 0.25)), 2, u, 4, 2, 2) is False
    # an expert of a dropped group (score 0.3125 - u/4) nearly ties the K-th
    # selected key 0.3125, but it is ineligible: harmless
    k = g4((0.5, 0.125), (0.3125, 0.1875), (0.3125 - u / 4,), (0.0625,))
    assert one(k, 2, u, 4, 2, 2) is False
    # the K-th eligible key and the next eligible one (in a kept group) nearly tie
    k = g4((0.5, 0.375), (0.375 - u / 2, 0.125), (), (0.0625,))
    assert one(k, 2, u, 4, 2, 2) is True


def pin_dense_capacity(seed=11):
    """Capacity drops in the forward pass: the layer equals the dense
    all-experts restatement with the gates of dropped pairs set to zero and the
    surviving gates left as they are.  The kept pairs are found here by walking
    the tokens in order with a counter per expert (the lowest token indices are
    admitted first); capacities for T*K = 80 rows over 6 experts are written
    out by hand: CF 1.0 -> 13, 0.5 -> 6, 0.001 -> 0 (every pair dropped, so
    y = h + the shared expert)."""
    rng = np.random.default_rng(seed)
    T, d, f, fs, E, K, Es = 40, 16, 24, 10, 6, 2, 1
    h = rng.normal(size=(T, d)).astype(F32)
    e = (rng.normal(size=(E, d)) * 0.5).astype(F32)
    e[0] += 1.0                                   # skewed: expert 0 overflows its capacity
    b = np.zeros(E, F32)
    W = [rng.normal(size=(E, f, d)), rng.normal(size=(E, f, d)), rng.normal(size=(E, d, f))]
    sW = [rng.normal(size=(Es, fs, d)), rng.normal(size=(Es, fs, d)), rng.normal(size=(Es, d, fs))]
    dropped_any = False
    for cf, C in ((1.0, 13), (0.5, 6), (0.001, 0)):
        cfg = mo.LayerConfig(T=T, d_model=d, E_r=E, E_s=Es, K=K, capacity_factor=cf)
        out = mo.layer_forward(cfg, h, e, b, mo.array_weights(*W, *sW))
        used = [0] * E
        G = np.zeros((T, E))
        for t in range(T):
            for k in range(K):
                i = int(out["idx"][t, k])
                if used[i] < C:
                    G[t, i] = float(out["gates"][t, k])
                    used[i] += 1
                else:
                    dropped_any = True
        want = _dense_layer(h.astype(np.float64), G, W, sW)
        assert np.allclose(out["y"], want, rtol=1e-11, atol=1e-11), cf
        assert out["kept"].tolist() == used, cf
        if C == 0:
            assert np.allclose(out["y"], _dense_layer(h.astype(np.float64), np.zeros((T, E)), W, sW),
                               rtol=1e-12, atol=1e-12)
    assert dropped_any


PINS = [pin_worked_bias_example, pin_bruteforce_topk, pin_bruteforce_grouped, pin_gates_properties,
        pin_counts_and_bias, pin_softmax_closed_form, pin_k_equals_e, pin_dense_reduction,
        pin_dense_all_experts, pin_capacity, pin_permutation_properties, pin_near_tie_bruteforce,
        pin_near_tie_handbuilt, pin_dense_capacity]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


def test_combinatorics_golden():
    g = _load("combinatorics.json")
    for n, k, want in g["choose"]:
        assert math.comb(n, k) == want
        if math.comb(n, k) < 200:
            assert sum(1 for _ in itertools.combinations(range(n), k)) == want
    for n, k, approx, rel in g["approx"]:
        assert abs(math.comb(n, k) - approx) <= rel * approx


# ---------------------------------------------------------------------------
# planted mistakes: each slip in the oracle must fail at least one pin
# ---------------------------------------------------------------------------

def _mut_bias_sign(b32, counts, K, T, gamma):
    E_r = counts.shape[0]
    sgn = np.sign(E_r * counts.astype(np.int64) - K * T).astype(F32)
    return (np.asarray(b32, F32) + F32(gamma) * sgn).astype(F32)


def _mut_sign_zero_up(b32, counts, K, T, gamma):
    E_r = counts.shape[0]
    sgn = np.where(E_r * counts.astype(np.int64) > K * T, -1.0, 1.0).astype(F32)
    return (np.asarray(b32, F32) + F32(gamma) * sgn).astype(F32)


def _mut_gates_biased(s32, idx):          # gates taken from the biased keys' order: no renorm
    return np.take_along_axis(s32.astype(F32), idx.astype(np.int64), axis=1)


def _mut_tie_high(s32, b32, K, n_groups=1, topk_groups=1, group_topn=0):
    keys = mo.selection_keys(s32, b32)
    elig = mo.eligible_mask(keys, n_groups, topk_groups, group_topn)
    masked = np.where(elig, keys, F32(-np.inf)).astype(F32)[:, ::-1]
    E = keys.shape[1]
    order = (E - 1) - np.argsort(-masked, axis=1, kind="stable")[:, :K]
    return np.sort(order, axis=1).astype(np.int32)


def _mut_capacity_ceil(T, K, E_r, capacity_factor):
    cf = float(np.float32(capacity_factor))
    return T * K if cf <= 0 else int(math.ceil(T * K * cf / E_r))


def _mut_swiglu_transposed(x, w_gate, w_up, w_down):
    x = np.asarray(x, np.float64)
    u = x @ np.asarray(w_gate, np.float64).T
    v = x @ np.asarray(w_up, np.float64).T
    a = u / (1.0 + np.exp(-u)) * v
    wd = np.asarray(w_down, np.float64)
    return a @ wd.reshape(wd.shape[1], wd.shape[0])        # wrong orientation of W_down


def _mut_silu_as_sigmoid(x, w_gate, w_up, w_down):
    x = np.asarray(x, np.float64)
    u = x @ np.asarray(w_gate, np.float64).T
    v = x @ np.asarray(w_up, np.float64).T
    return (1.0 / (1.0 + np.exp(-u)) * v) @ np.asarray(w_down, np.float64).T


def _mut_group_sum_top1(keys, n_groups, group_topn):
    T, E = keys.shape
    return -np.sort(-keys.reshape(T, n_groups, E // n_groups), axis=2)[:, :, 0].astype(F32)


def _mut_selection_ignores_bias(s32, b32):
    return s32.astype(F32)


def _mut_counts_kept_only(idx, E_r):      # off-by-one histogram
    c = np.bincount(idx.reshape(-1).astype(np.int64), minlength=E_r + 1)[1:E_r + 1]
    return np.concatenate([c, np.zeros(max(0, E_r - len(c)), np.int64)]).astype(np.int64)


def _near_tie_variant(s32, b32, K, n_groups, topk_groups, group_topn, gap, *, kth=None, masked=True,
                      sort_groups=True, groups=True):
    keys = mo.selection_keys(s32, b32).astype(np.float64)
    T, E = keys.shape
    fragile = np.zeros(T, dtype=bool)
    if groups and n_groups > 1 and group_topn > 0 and topk_groups < n_groups:
        G = mo.group_scores(mo.selection_keys(s32, b32), n_groups, group_topn).astype(np.float64)
        if sort_groups:
            G = np.sort(G, axis=1)[:, ::-1]
        fragile |= (G[:, topk_groups - 1] - G[:, topk_groups]) < gap
    elig = mo.eligible_mask(mo.selection_keys(s32, b32), n_groups, topk_groups, group_topn)
    srt = -np.sort(-(np.where(elig, keys, -np.inf) if masked else keys), axis=1)
    k = K if kth is None else kth
    if 1 <= k < E:
        nxt = srt[:, k]
        fragile |= np.isfinite(nxt) & ((srt[:, k - 1] - nxt) < gap)
    return fragile


def _mut_near_tie_gap_after_k(s32, b32, K, n_groups=1, topk_groups=1, group_topn=0, gap=1e-5):
    return _near_tie_variant(s32, b32, K, n_groups, topk_groups, group_topn, gap, kth=K + 1)


def _mut_near_tie_gap_inside(s32, b32, K, n_groups=1, topk_groups=1, group_topn=0, gap=1e-5):
    return _near_tie_variant(s32, b32, K, n_groups, topk_groups, group_topn, gap, kth=K - 1)


def _mut_near_tie_unmasked(s32, b32, K, n_groups=1, topk_groups=1, group_topn=0, gap=1e-5):
    return _near_tie_variant(s32, b32, K, n_groups, topk_groups, group_topn, gap, masked=False)


def _mut_near_tie_groups_unsorted(s32, b32, K, n_groups=1, topk_groups=1, group_topn=0, gap=1e-5):
    return _near_tie_variant(s32, b32, K, n_groups, topk_groups, group_topn, gap, sort_groups=False)


def _mut_near_tie_no_group_gap(s32, b32, K, n_groups=1, topk_groups=1, group_topn=0, gap=1e-5):
    return _near_tie_variant(s32, b32, K, n_groups, topk_groups, group_topn, gap, groups=False)


def _mut_layer_output_ignores_drops(cfg, h, idx, gates, disp, weights, tokens=None):
    full = mo.Dispatch(disp.counts, disp.counts, disp.offsets, disp.perm_tok, disp.perm_slot,
                       np.zeros_like(disp.row_of))
    return _orig_layer_output(cfg, h, idx, gates, full, weights, tokens)


def _mut_layer_output_renormalises(cfg, h, idx, gates, disp, weights, tokens=None):
    kept = disp.row_of >= 0
    g = np.where(kept, gates, 0).astype(np.float64)
    ssum = g.sum(1, keepdims=True)
    g = np.where(ssum > 0, g / np.where(ssum > 0, ssum, 1), 0).astype(F32)
    return _orig_layer_output(cfg, h, idx, g, disp, weights, tokens)


_orig_layer_output = mo.layer_output


MUTATIONS = [
    ("bias_update", _mut_bias_sign),
    ("bias_update", _mut_sign_zero_up),
    ("gates_from_scores", _mut_gates_biased),
    ("select_experts", _mut_tie_high),
    ("capacity", _mut_capacity_ceil),
    ("swiglu", _mut_swiglu_transposed),
    ("swiglu", _mut_silu_as_sigmoid),
    ("group_scores", _mut_group_sum_top1),
    ("selection_keys", _mut_selection_ignores_bias),
    ("load_counts", _mut_counts_kept_only),
    ("near_tie_tokens", _mut_near_tie_gap_after_k),
    ("near_tie_tokens", _mut_near_tie_gap_inside),
    ("near_tie_tokens", _mut_near_tie_unmasked),
    ("near_tie_tokens", _mut_near_tie_groups_unsorted),
    ("near_tie_tokens", _mut_near_tie_no_group_gap),
    ("layer_output", _mut_layer_output_ignores_drops),
    ("layer_output", _mut_layer_output_renormalises),
]


@pytest.mark.parametrize("name,mut", MUTATIONS, ids=[m[1].__name__ for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, mut):
    monkeypatch.setattr(mo, name, mut)
    failed = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake in {name} was not caught by any pin"

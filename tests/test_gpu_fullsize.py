"""Full-size workloads in the launch configuration bench.py times.

Routing is checked on every token (fed with the oracle's fp32 scores: bit-exact;
with the GPU's own logits: identical outside the 1e-5 near-tie set).  Layer
outputs are checked on a few sampled tokens, for which the oracle evaluates the
experts in float64 from weights regenerated on the host by the generator's C
twin (the device copy comes from its CUDA twin; both equal the numpy
definition bit for bit).
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as mo
from gpu_helpers import (BF16_TOL, Layer, LazyHostWeights, check_close, device_weights, oracle_cfg,
                         out_eps_of, to_dev, torch_dtype)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

FULL = ["mixtral_8x14336", "finegrained_64x1408", "finegrained_64x1408_cf1.25", "deepseek_v3",
        "deepseek_v3_decode"]
N_SAMPLE = 3


def _sample_tokens(w, fragile, seed=7):
    rng = np.random.default_rng(seed)
    ok = np.nonzero(~fragile)[0]
    return np.sort(rng.choice(ok, size=min(N_SAMPLE, len(ok)), replace=False))


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
    tok = _sample_tokens(w, np.zeros(w.T, bool))
    # a token whose every expert was dropped must still be sampled when it exists
    if w.capacity_factor > 0:
        dropped = np.nonzero((disp.row_of < 0).any(axis=1))[0]
        if len(dropped):
            tok = np.unique(np.concatenate([tok, dropped[:1]]))
    y_ref = mo.layer_output(cfg, h, idx, gates, disp, LazyHostWeights(w).source(), tokens=tok)
    check_close(y.float().cpu().numpy()[tok], y_ref, h[tok], BF16_TOL, True, out_eps_of(w))


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
            tok = _sample_tokens(w, np.zeros(w.T, bool), seed=step)
            y_ref = mo.layer_output(cfg, h, idx, gates, disp, src, tokens=tok)
            check_close(y.float().cpu().numpy()[tok], y_ref, h[tok], BF16_TOL, True, 2.0 ** -8)
    assert L.device_error() == 0

"""Layer backward on the GPU (moe_layer_backward after a train = 1 forward)
against the oracle's layer_backward: dL/dh, dL/de and every expert weight
gradient, for the routing the forward chose (the oracle's fp32 scores are fed
to both, so the selections agree bit for bit).

The GPU path keeps U, V, A, dO, dU, dV and dX in bf16 and accumulates in fp32,
so each gradient carries a few bf16 roundings (a CPU simulation of those
roundings reproduces the GPU's error on the weight gradients to every printed
digit).  The bar, per tensor (per expert for the weights), is the
rounding-aware one of the forward: max(|grad - ref| - 2^-8 |ref|) <= 3e-2 *
RMS(ref), the 2^-8 |ref| term allowing the stored bf16 value's own rounding;
experts without kept rows must get exactly zero."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as mo
import sparse_mixture_experts_selection_b200 as moe
from gpu_helpers import HostWeights, oracle_cfg, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

W = mi.WORKLOADS
TOL = 3e-2
CASES = {
    "deepseek_small": W["deepseek_v3"].with_(T=520, d_model=256, E_r=64, E_s=1, K=6, d_ffn=256,
                                             d_ffn_shared=384, n_groups=8, topk_groups=3),
    "finegrained_near_tile": W["finegrained_64x1408"].with_(T=440, d_model=192, E_r=16, E_s=2, K=4,
                                                           d_ffn=192, d_ffn_shared=128),
    # capacity 1.0: some (token, expert) pairs are dropped
    "finegrained_cf": W["finegrained_64x1408_cf1.25"].with_(T=600, d_model=192, E_r=16, E_s=2, K=4,
                                                            d_ffn=192, d_ffn_shared=128, capacity_factor=1.0),
    "mixtral_small": W["mixtral_8x14336"].with_(T=300, d_model=256, d_ffn=320),
}


def _close(got, ref, what):
    ref = np.asarray(ref, np.float64)
    got = np.asarray(got, np.float64)
    assert np.all(np.isfinite(got)), what
    scale = np.sqrt(np.mean(ref ** 2))
    err = np.max(np.abs(got - ref) - 2.0 ** -8 * np.abs(ref)) if ref.size else 0.0
    assert err <= TOL * scale, (what, err, scale)


def run_backward(w, seed=7):
    h, e, b = mi.gen_h(w, 0), mi.gen_centroids(w), mi.gen_bias(w)
    HW = HostWeights(w)
    cfg_o = oracle_cfg(w)
    s = mo.affinity(h, e, w.score_fn)
    b_sel = b if w.score_fn == 0 else np.zeros(w.E_r, np.float32)
    idx, gates, disp = mo.route(cfg_o, s, b_sel)
    rng = np.random.default_rng(seed)
    dy = mi.round_bf16(rng.normal(size=(w.T, w.d_model)).astype(np.float32))
    ref = mo.layer_backward(cfg_o, h, e, s, idx, gates, disp, HW.source(), dy)

    cfg = moe.config_for(w, train=1)
    Wd = HW.device()
    ws = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    hd, ed, bd, sd = to_dev(h, torch.bfloat16), to_dev(e), to_dev(b), to_dev(s)
    y = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    idx_d = torch.empty((w.T, w.K), dtype=torch.int32, device="cuda")
    moe.moe_layer_forward(cfg, hd, ed, bd, Wd["gate"], Wd["up"], Wd["down"], Wd["sgate"], Wd["sup"], Wd["sdown"],
                          y, ws, s_in=sd, idx_out=idx_d)
    dh = torch.empty_like(hd)
    de = torch.empty((w.E_r, w.d_model), dtype=torch.float32, device="cuda")
    G = {k: (torch.full_like(v, 7.0) if v is not None else None) for k, v in Wd.items()}
    moe.moe_layer_backward(cfg, hd, ed, sd, idx_d, Wd["gate"], Wd["up"], Wd["down"], Wd["sgate"], Wd["sup"],
                           Wd["sdown"], to_dev(dy, torch.bfloat16), dh, de, G["gate"], G["up"], G["down"],
                           G["sgate"], G["sup"], G["sdown"], ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    assert np.array_equal(idx_d.cpu().numpy(), idx)
    return ref, dh.float().cpu().numpy(), de.cpu().numpy(), {k: (v.float().cpu().numpy() if v is not None else None)
                                                             for k, v in G.items()}


@pytest.mark.parametrize("name", sorted(CASES))
def test_layer_backward_matches_oracle(name):
    w = CASES[name]
    ref, dh, de, G = run_backward(w)
    _close(dh, ref["dh"], "dh")
    _close(de, ref["de"], "de")
    for which in ("gate", "up", "down"):
        for ex in range(w.E_r):
            key = (which, ex)
            if key in ref["grads"]:
                _close(G[which][ex], ref["grads"][key], key)
            else:
                assert np.all(G[which][ex] == 0), key          # no kept rows: zero gradient
    for j in range(w.E_s):
        for which in ("sgate", "sup", "sdown"):
            _close(G[which][j], ref["grads"][(which, j)], (which, j))


EDGE = {
    "single_token": CASES["deepseek_small"].with_(T=1),
    "dense_E1_K1": CASES["finegrained_near_tile"].with_(E_r=1, K=1),
    "no_residual": CASES["finegrained_near_tile"].with_(add_residual=0),
    # Zipf-skewed centroids: the hottest experts hold two full row tiles and a merged tail
    "hot_expert": CASES["deepseek_small"].with_(T=700, centroid_skew="zipf_1.2"),
    # more experts than selections: many experts without rows (zero weight gradients)
    "sparse_experts": CASES["deepseek_small"].with_(T=40),
}


@pytest.mark.parametrize("name", sorted(EDGE))
def test_layer_backward_edge_cases(name):
    w = EDGE[name]
    ref, dh, de, G = run_backward(w)
    _close(dh, ref["dh"], "dh")
    if np.any(ref["de"] != 0):
        _close(de, ref["de"], "de")
    else:                                   # one softmax expert: the gate is 1 whatever z is
        assert np.max(np.abs(de)) <= 1e-6
    for which in ("gate", "up", "down"):
        for ex in range(w.E_r):
            key = (which, ex)
            if key in ref["grads"]:
                _close(G[which][ex], ref["grads"][key], key)
            else:
                assert np.all(G[which][ex] == 0), key
    for j in range(w.E_s):
        for which in ("sgate", "sup", "sdown"):
            _close(G[which][j], ref["grads"][(which, j)], (which, j))


def test_backward_rejects_inference_config():
    w = CASES["deepseek_small"]
    cfg = moe.config_for(w)                                  # train = 0
    ws = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.moe_layer_backward(cfg, x, x, x, x, x, x, x, x, x, x, x, x, x, x, x, x, x, x, x, ws)

"""Layer backward on the GPU (moe_layer_backward after a train = 1 forward)
against the oracle's layer_backward: dL/dh, dL/de and every expert weight
gradient, for the routing the forward chose (the oracle's fp32 scores are fed
to both, so the selections agree bit for bit).

The GPU path keeps U, V, A, dO, dU, dV and dX in bf16 and accumulates in fp32,
so each gradient carries a few bf16 roundings.  The bar (normwise and
elementwise, backward_cases) sits above the error of a float64 model that
rounds to bf16 at exactly those points (bf16_backward_model; its distance from
the oracle is checked against the bar on the CPU).  Experts without kept rows
must get exactly zero."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as mo
import sparse_mixture_experts_selection_b200 as moe
import backward_cases as bc
import bf16_backward_model as bm
from gpu_helpers import HostWeights, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

CASES, EDGE = bc.CASES, bc.EDGE


def run_backward(w, seed=7):
    cfg_o, h, e, b, s, idx, gates, disp, dy = bc.inputs(w, seed)
    HW = HostWeights(w)
    ref = mo.layer_backward(cfg_o, h, e, s, idx, gates, disp, HW.source(), dy)
    ref["model"] = bm.layer_backward_bf16(cfg_o, h, e, s, idx, gates, disp, HW.source(), dy)

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


def _check_all(w, ref, dh, de, G):
    model = ref["model"]
    bc.check(dh, ref["dh"], "dh")
    bc.check_model(dh, model["dh"], "dh")
    if np.any(ref["de"] != 0):
        bc.check(de, ref["de"], "de")
        bc.check_model(de, model["de"], "de")
    else:                                   # one expert: the gate is 1 whatever z is
        assert np.max(np.abs(de)) <= 1e-6
    for what, got, r in bc.each_gradient(w, ref, G):
        bc.check(got, r, what)
        bc.check_model(got, model["grads"][what], what)


@pytest.mark.parametrize("name", sorted(CASES))
def test_layer_backward_matches_oracle(name):
    w = CASES[name]
    _check_all(w, *run_backward(w))


@pytest.mark.parametrize("name", sorted(EDGE))
def test_layer_backward_edge_cases(name):
    w = EDGE[name]
    _check_all(w, *run_backward(w))


def test_backward_rejects_inference_config():
    w = CASES["deepseek_small"]
    cfg = moe.config_for(w)                                  # train = 0
    ws = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.moe_layer_backward(cfg, x, x, x, x, x, x, x, x, x, x, x, x, x, x, x, x, x, x, x, ws)

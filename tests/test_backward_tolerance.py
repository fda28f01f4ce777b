"""The backward parity bar against the error the bf16 storage points alone
cause: the bf16 storage model (same float64 arithmetic as the oracle, rounded
to bf16 where the GPU path stores bf16) must sit well inside the bar on every
backward parity case, and the bar must not be so loose that a dropped term
passes."""
import numpy as np
import pytest

import backward_cases as bc
import bf16_backward_model as bm
from gpu_helpers import HostWeights
from oracle import moe_oracle as mo

ALL = dict(bc.CASES, **bc.EDGE)


def _both(w):
    cfg, h, e, b, s, idx, gates, disp, dy = bc.inputs(w)
    src = HostWeights(w).source()
    ref = mo.layer_backward(cfg, h, e, s, idx, gates, disp, src, dy)
    model = bm.layer_backward_bf16(cfg, h, e, s, idx, gates, disp, src, dy)
    return ref, model


@pytest.mark.parametrize("name", ["deepseek_small", "single_token", "hot_expert", "sparse_experts",
                                  "finegrained_cf", "dense_E1_K1", "softmax_dropped"])
def test_bf16_model_within_three_quarters_of_the_bar(name):
    w = ALL[name]
    ref, model = _both(w)
    worst_n = worst_m = 0.0
    for what in ("dh", "de"):
        if np.any(ref[what] != 0):
            n, m = bc.errors(model[what], ref[what])
            worst_n, worst_m = max(worst_n, n), max(worst_m, m)
    G = {k: {ex: model["grads"].get((k, ex), np.zeros(1)) for ex in range(max(w.E_r, w.E_s))}
         for k in ("gate", "up", "down", "sgate", "sup", "sdown")}
    for what, got, r in bc.each_gradient(w, ref, G):
        n, m = bc.errors(got, r)
        worst_n, worst_m = max(worst_n, n), max(worst_m, m)
    assert worst_n <= 0.75 * bc.NORM_TOL, worst_n
    assert worst_m <= 0.75 * bc.ELEM_TOL, worst_m
    assert worst_n > 1e-3            # the model does round: it is not the oracle again


def test_bar_catches_a_dropped_term():
    # the SiLU'(u) factor's second term dropped from dU (a plausible slip) moves
    # the gate-weight gradients far outside the bar
    w = bc.CASES["deepseek_small"]
    cfg, h, e, b, s, idx, gates, disp, dy = bc.inputs(w)
    src = HostWeights(w).source()
    ref = mo.layer_backward(cfg, h, e, s, idx, gates, disp, src, dy)
    ex = int(idx[0, 0])
    rows, ks = np.nonzero((idx == ex) & (disp.row_of >= 0))
    x = h[rows].astype(np.float64)
    g = gates[rows, ks].astype(np.float64)[:, None]
    wg, wu, wd = (np.asarray(src(k, ex), np.float64) for k in ("gate", "up", "down"))
    u, v = x @ wg.T, x @ wu.T
    sig = 1.0 / (1.0 + np.exp(-u))
    du_wrong = ((g * dy[rows]) @ wd) * v * sig          # SiLU'(u) taken as sig alone
    n, m = bc.errors(du_wrong.T @ x, ref["grads"][("gate", ex)])
    assert n > 10 * bc.NORM_TOL and m > bc.ELEM_TOL

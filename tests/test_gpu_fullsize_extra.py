"""Full-size checks of the e4m3-weight layer and of the layer backward, in the
launch configuration bench.py times (DeepSeek-V3 shapes, T = 4096 and 64),
on sampled outputs the oracle can evaluate one by one: a few tokens' y (e4m3),
a few tokens' dL/dh and whole weight gradients of two experts (backward).
Routing is fed with the oracle's fp32 scores, so it agrees bit for bit."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import sparse_mixture_experts_selection_b200 as moe
from oracle import moe_oracle as mo
import backward_cases as bc
from gpu_helpers import BF16_TOL, LazyHostWeights, check_close, device_weights, oracle_cfg, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


def _routing(w):
    h, e, b = mi.gen_h(w), mi.gen_centroids(w), mi.gen_bias(w)
    s = mo.affinity(h, e, w.score_fn)
    b_sel = b if w.score_fn == 0 else np.zeros(w.E_r, np.float32)
    idx, gates, disp = mo.route(oracle_cfg(w), s, b_sel)
    return h, e, b, s, idx, gates, disp


@pytest.mark.parametrize("name", ["deepseek_v3_e4m3", "deepseek_v3_decode_e4m3"])
def test_fullsize_e4m3_sampled_outputs(name):
    w = mi.WORKLOADS[name]
    h, e, b, s, idx, gates, disp = _routing(w)
    W = device_weights(w)                               # the bf16 weights (generator's CUDA twin)
    Q = {}
    for k, t in W.items():
        if t is None:
            Q[k] = None
            continue
        n, r, c = t.shape
        Q[k] = torch.empty(moe.moe_quantized_bytes(n * r, c), dtype=torch.uint8, device="cuda")
        moe.moe_quantize_rows(t, moe.DTYPE_BF16, n * r, c, Q[k])
    del W
    torch.cuda.synchronize()
    cfg = moe.config_for(w)
    ws = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    y = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    idx_d = torch.empty((w.T, w.K), dtype=torch.int32, device="cuda")
    moe.moe_layer_forward(cfg, to_dev(h, torch.bfloat16), to_dev(e), to_dev(b), Q["gate"], Q["up"], Q["down"],
                          Q["sgate"], Q["sup"], Q["sdown"], y, ws, s_in=to_dev(s), idx_out=idx_d)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    assert np.array_equal(idx_d.cpu().numpy(), idx)
    # the device blob of one expert's W_gate rows equals the oracle's quantization of them
    lw = LazyHostWeights(w)
    ex0 = int(idx[0, 0])
    f, d = w.d_ffn, w.d_model
    blob = Q["gate"].cpu().numpy()
    codes = blob[ex0 * f * d:(ex0 + 1) * f * d].reshape(f, d)
    scales = blob[w.E_r * f * d:].view(np.float32)[ex0 * f:(ex0 + 1) * f]
    want_c, want_s = mo.quantize_rows(lw.get("gate", ex0))
    assert np.array_equal(codes, want_c) and np.array_equal(scales.view(np.int32), want_s.view(np.int32))
    # sampled tokens' outputs against the oracle's quantized layer
    tok = np.sort(np.random.default_rng(3).choice(w.T, size=2, replace=False))
    qcache = {}

    def q8(which, ex):
        key = (which, int(ex))
        if key not in qcache:
            qcache[key] = mo.quantize_rows(lw.get(which, int(ex)))
        return qcache[key]
    y_ref = mo.layer_output_q8(oracle_cfg(w), h, idx, gates, disp, q8, tokens=tok)
    check_close(y.float().cpu().numpy()[tok], y_ref, h[tok], BF16_TOL, True, 2.0 ** -8)


def test_fullsize_backward_sampled():
    w = mi.WORKLOADS["deepseek_v3"]
    h, e, b, s, idx, gates, disp = _routing(w)
    W = device_weights(w)
    G = {k: (torch.empty_like(t) if t is not None else None) for k, t in W.items()}
    cfg = moe.config_for(w, train=1)
    ws = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    hd, ed, sd = to_dev(h, torch.bfloat16), to_dev(e), to_dev(s)
    y = torch.empty_like(hd)
    idx_d = torch.empty((w.T, w.K), dtype=torch.int32, device="cuda")
    moe.moe_layer_forward(cfg, hd, ed, to_dev(b), W["gate"], W["up"], W["down"], W["sgate"], W["sup"],
                          W["sdown"], y, ws, s_in=sd, idx_out=idx_d)
    dy = mi.round_bf16(np.random.default_rng(11).normal(size=(w.T, w.d_model)).astype(np.float32))
    dh = torch.empty_like(hd)
    de = torch.empty((w.E_r, w.d_model), dtype=torch.float32, device="cuda")
    moe.moe_layer_backward(cfg, hd, ed, sd, idx_d, W["gate"], W["up"], W["down"], W["sgate"], W["sup"],
                           W["sdown"], to_dev(dy, torch.bfloat16), dh, de, G["gate"], G["up"], G["down"],
                           G["sgate"], G["sup"], G["sdown"], ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    assert np.array_equal(idx_d.cpu().numpy(), idx)
    lw = LazyHostWeights(w)
    kept = disp.row_of >= 0
    # whole weight gradients of the busiest expert and of one more
    counts = disp.kept
    rng = np.random.default_rng(5)
    for ex in [int(np.argmax(counts)), int(rng.choice(np.nonzero(counts > 0)[0]))]:
        rows, ks = np.nonzero((idx == ex) & kept)
        g = gates[rows, ks].astype(np.float64)[:, None]
        _, dwg, dwu, dwd, _ = mo.swiglu_backward(h[rows], lw.get("gate", ex), lw.get("up", ex),
                                                 lw.get("down", ex), g * dy[rows])
        for which, ref in (("gate", dwg), ("up", dwu), ("down", dwd)):
            bc.check(G[which][ex].float().cpu().numpy(), ref, (which, ex))
    # dL/dh of two sampled tokens: residual, shared expert, routed experts, router
    dh_g = dh.float().cpu().numpy()
    for t in np.sort(rng.choice(w.T, size=2, replace=False)):
        x = h[t:t + 1]
        acc = dy[t].astype(np.float64) * w.add_residual
        for j in range(w.E_s):
            dx, *_ = mo.swiglu_backward(x, lw.get("sgate", j), lw.get("sup", j), lw.get("sdown", j), dy[t:t + 1])
            acc = acc + dx[0]
        dg = np.zeros((1, w.K))
        for k in range(w.K):
            ex = int(idx[t, k])
            dx, _, _, _, o = mo.swiglu_backward(x, lw.get("gate", ex), lw.get("up", ex), lw.get("down", ex),
                                                float(gates[t, k]) * dy[t:t + 1])
            acc = acc + dx[0]
            dg[0, k] = float((dy[t].astype(np.float64) * o[0]).sum())
        dz = mo.score_backward(s[t:t + 1], mo.gate_backward(s[t:t + 1], idx[t:t + 1], dg), w.score_fn)
        acc = acc + (dz @ e.astype(np.float64))[0]
        bc.check(dh_g[t], acc, ("dh", int(t)))

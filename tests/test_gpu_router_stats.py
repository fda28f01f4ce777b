"""Router losses and logging on the GPU (moe_router_stats, and the fp32 logits
that moe_route / moe_layer_forward export for the z-loss) against the oracle.

The statistics are fed the oracle's scores, logits, selections and kept
counts, so every difference is the GPU's reduction error: the bar is a
relative 1e-5 (fp32 partial sums of at most a few thousand terms, finished in
fp64), MaxVio exactly.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as mo
import sparse_mixture_experts_selection_b200 as moe
from gpu_helpers import HostWeights, Layer, to_dev, torch_dtype

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

W = mi.WORKLOADS
REL = 1e-5

STATS_CASES = [
    # (T, E, K, score_fn, seq_len, capacity_factor, with_z)
    (1000, 64, 8, 0, 0, 0.0, True),
    (4096, 256, 8, 0, 512, 1.25, True),      # DeepSeek-V3 routing shape, 8 sequences
    (513, 8, 2, 1, 171, 1.0, True),          # softmax; 171 = 2 chunks of 64 + a ragged 43
    (333, 1024, 16, 0, 1, 0.0, False),       # widest shape, one-token sequences, no logits
    (1, 4, 1, 1, 1, 0.0, True),              # single token
    (640, 16, 16, 0, 640, 0.5, True),        # K = E_r: uniform load, heavy dropping
]


def _stats_gpu(T, E, K, fn, s, z, idx, kept, seq_len, a_aux, c_z, a_seq):
    cfg = moe.MoeConfig(T=T, d_model=64, E_r=E, E_s=0, K=K, d_ffn=64, d_ffn_shared=0, score_fn=fn,
                        n_groups=1, topk_groups=1, group_topn=0, capacity_factor=0.0, dtype=0,
                        add_residual=1)
    ws = moe.alloc_workspace(moe.moe_router_stats_workspace_size(cfg, seq_len))
    out = torch.full((6,), float("nan"), dtype=torch.float32, device="cuda")
    moe.moe_router_stats(cfg, to_dev(s), None if z is None else to_dev(z),
                         to_dev(idx, torch.int32), None if kept is None else to_dev(kept, torch.int32),
                         out, ws, seq_len=seq_len, alpha_aux=a_aux, c_z=c_z, alpha_seq=a_seq)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("case", STATS_CASES, ids=[str(c) for c in STATS_CASES])
def test_router_stats_match_oracle(case):
    T, E, K, fn, seq_len, cf, with_z = case
    rng = np.random.default_rng(T + 13 * E + K)
    # logits with a per-expert skew, so that the load is uneven and the losses
    # sit away from their minima
    z = (rng.normal(size=(T, E)) * 2 + np.linspace(-1, 1, E)).astype(np.float32)
    s = mo.sigmoid_scores(z) if fn == 0 else mo.softmax_scores(z)
    idx = mo.select_experts(s, np.zeros(E, np.float32), K)
    disp = mo.dispatch(idx, E, cf)
    kept = disp.kept if cf > 0 else None
    a_aux, c_z, a_seq = 0.01, 1e-3, 1e-4
    got = _stats_gpu(T, E, K, fn, s, z if with_z else None, idx, kept, seq_len, a_aux, c_z, a_seq)
    counts = mo.load_counts(idx, E)
    want = np.array([
        mo.aux_loss(s, idx, E, K, a_aux),
        mo.z_loss(z, c_z) if with_z else 0.0,
        mo.seq_balance_loss(s, idx, E, K, seq_len, a_seq) if seq_len else 0.0,
        mo.load_entropy(counts),
        mo.max_vio(counts, K, T, E),
        mo.dropped_rate(kept, counts) if kept is not None else 0.0,
    ])
    names = moe.ROUTER_STATS
    for i, n in enumerate(names):
        assert abs(got[i] - want[i]) <= REL * abs(want[i]) + 1e-7, (n, got[i], want[i])
    assert np.float32(got[4]) == np.float32(want[4])     # MaxVio: integer counts, exact


def test_router_stats_reject_bad_seq_len():
    cfg = moe.MoeConfig(T=100, d_model=64, E_r=8, E_s=0, K=2, d_ffn=64, d_ffn_shared=0, score_fn=0,
                        n_groups=1, topk_groups=1, group_topn=0, capacity_factor=0.0, dtype=0,
                        add_residual=1)
    with pytest.raises(moe.MoeError):
        moe.moe_router_stats_workspace_size(cfg, 30)


@pytest.mark.parametrize("name", ["toy_fp32", "deepseek_small"])
def test_exported_logits_match_oracle(name):
    """z_out of moe_route and of moe_layer_forward: the fp32 logits h_t . e_i
    (tensor-core split-K for bf16 layers, CUDA cores for fp32), within a few
    fp32 ulps of the double-accumulated value; both entry points agree bit for
    bit."""
    if name == "toy_fp32":
        w = W["toy_fp32"].with_(steps=1)
    else:
        w = W["deepseek_v3"].with_(T=520, d_model=256, E_r=64, E_s=1, K=6, d_ffn=256,
                                   d_ffn_shared=384, n_groups=8, topk_groups=3)
    h, e, b = mi.gen_h(w, 0), mi.gen_centroids(w), mi.gen_bias(w)
    z_ref = mo.router_logits(h, e).astype(np.float64)
    cfg = moe.config_for(w)
    T, K, E = w.T, w.K, w.E_r
    ws = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    gates = torch.empty((T, K), dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    z_route = torch.empty((T, E), dtype=torch.float32, device="cuda")
    hd, ed, bd = to_dev(h, torch_dtype(w)), to_dev(e), to_dev(b)
    moe.moe_route(cfg, hd, ed, bd, None, None, idx, gates, counts, ws, z_out=z_route)
    L = Layer(w, HostWeights(w).device())
    L.forward(hd, ed, bd)
    assert L.device_error() == 0
    zr = z_route.cpu().numpy()
    zl = L.z.cpu().numpy()
    assert np.array_equal(zr.view(np.int32), zl.view(np.int32))
    scale = max(1.0, float(np.max(np.abs(z_ref))))
    assert np.max(np.abs(zr.astype(np.float64) - z_ref)) <= 4e-6 * scale

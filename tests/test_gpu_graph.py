"""The layer forward captured in a CUDA graph.  moe_layer_forward only
enqueues work on the caller's stream (kernels launched with programmatic
dependent launch, cluster launches for the CTA-pair GEMMs, a memset, no host
synchronisation, no allocation), so a caller can capture a whole step --
routing, dispatch, both grouped GEMMs, combine and the bias step -- once and
replay it.  Replays must match eager calls bit for bit, step after step,
including the carried bias."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import sparse_mixture_experts_selection_b200 as moe
from gpu_helpers import HostWeights, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


@pytest.mark.parametrize("name", ["deepseek_v3", "mixtral_8x14336", "mixtral_8x14336_pairs"])
def test_layer_forward_graph_replay_matches_eager(name):
    base = name.replace("_pairs", "")
    w = mi.WORKLOADS[base].with_(T=256, d_model=256, d_ffn=256, d_ffn_shared=128,
                                  E_r=min(mi.WORKLOADS[base].E_r, 32))
    if w.n_groups > 1:
        w = w.with_(n_groups=8, topk_groups=4)
    if name.endswith("_pairs"):
        # >= 512 rows per expert: the CTA-pair GEMMs (cluster launches), whose
        # units are claimed dynamically -- replays must still match bit for bit
        w = w.with_(T=2304)
        assert moe.moe_expert_ffn_tile_rows(moe.config_for(w), w.E_r, w.T * w.K) == 256
    Wd = HostWeights(w).device()
    e = to_dev(mi.gen_centroids(w))
    b0 = mi.gen_bias(w)
    steps = 3
    hs = [to_dev(mi.gen_h(w, s), torch.bfloat16) for s in range(steps)]
    cfg = moe.config_for(w)
    gamma = 0.01 if w.score_fn == 0 else 0.0

    def run(ws, h_in, b, y, idx):
        moe.moe_layer_forward(cfg, h_in, e, b, Wd["gate"], Wd["up"], Wd["down"], Wd["sgate"], Wd["sup"],
                              Wd["sdown"], y, ws, idx_out=idx, update_bias=gamma > 0, gamma=gamma)

    # eager reference
    ws_e = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    b_e = to_dev(b0)
    ref = []
    for s in range(steps):
        y = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
        idx = torch.empty((w.T, w.K), dtype=torch.int32, device="cuda")
        run(ws_e, hs[s], b_e, y, idx)
        torch.cuda.synchronize()
        ref.append((y.clone(), idx.clone(), b_e.clone()))
    assert moe.moe_get_device_error(ws_e) == 0

    # one step captured (static input/output buffers), replayed once per batch
    ws_g = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    b_g = to_dev(b0)
    h_st = torch.empty_like(hs[0])
    y_st = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    idx_st = torch.empty((w.T, w.K), dtype=torch.int32, device="cuda")
    # one eager call first (one-time setup of the library's kernels), on a
    # throw-away bias so the carried bias starts from b0 again
    h_st.copy_(hs[0])
    run(ws_g, h_st, to_dev(b0), y_st, idx_st)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run(ws_g, h_st, b_g, y_st, idx_st)
    for s in range(steps):
        h_st.copy_(hs[s])
        graph.replay()
        torch.cuda.synchronize()
        y_r, idx_r, b_r = ref[s]
        assert torch.equal(idx_st, idx_r), s
        assert torch.equal(y_st.view(torch.int16), y_r.view(torch.int16)), s
        assert torch.equal(b_g.view(torch.int32), b_r.view(torch.int32)), s
    assert moe.moe_get_device_error(ws_g) == 0
    del graph

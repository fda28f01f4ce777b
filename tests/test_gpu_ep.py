"""Expert-parallel layer on one GPU with the loopback exchange (W ranks in one
process, the rows moved by device copies): every rank's output against the
oracle's layer on that rank's tokens, routing bit-exact (scores fed), and the
bias step on the loads summed over the ranks bit-exact."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as mo
import sparse_mixture_experts_selection_b200 as moe
from sparse_mixture_experts_selection_b200 import ep
from gpu_helpers import BF16_TOL, HostWeights, check_close, oracle_cfg, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


@pytest.mark.parametrize("W,E_s", [(4, 1), (2, 0)])
def test_expert_parallel_loopback_matches_oracle(W, E_s):
    w = mi.WORKLOADS["deepseek_v3"].with_(T=96, d_model=128, E_r=16, E_s=E_s, K=4, d_ffn=128,
                                          d_ffn_shared=128, n_groups=4, topk_groups=2, group_topn=2)
    HW = HostWeights(w)
    Wd = HW.device()
    e, b = mi.gen_centroids(w), mi.gen_bias(w) + np.float32(0.003) * np.arange(w.E_r, dtype=np.float32)
    E_loc = w.E_r // W
    cfg = moe.config_for(w)
    layers = [ep.ExpertParallelLayer(cfg, r, W, to_dev(e), Wd["gate"][r * E_loc:(r + 1) * E_loc],
                                     Wd["up"][r * E_loc:(r + 1) * E_loc], Wd["down"][r * E_loc:(r + 1) * E_loc],
                                     Wd["sgate"], Wd["sup"], Wd["sdown"]) for r in range(W)]
    hs = [mi.gen_h(w, step) for step in range(W)]                # each rank its own tokens
    ss = [mo.affinity(h, e, w.score_fn) for h in hs]
    bd = to_dev(b)
    ys = [torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda") for _ in range(W)]
    mv = torch.empty(1, dtype=torch.float32, device="cuda")
    ep.forward(layers, [to_dev(h, torch.bfloat16) for h in hs], bd, ys, ep.LoopbackExchange(W), gamma=0.01,
               update_bias=True, max_vio=mv, s_in=[to_dev(s) for s in ss])
    torch.cuda.synchronize()
    counts = np.zeros(w.E_r, np.int64)
    for r in range(W):
        ref = mo.layer_forward(oracle_cfg(w), hs[r], e, b, HW.source(), s_in=ss[r])
        assert np.array_equal(layers[r].idx.cpu().numpy(), ref["idx"])
        check_close(ys[r].float().cpu().numpy(), ref["y"], hs[r], BF16_TOL, True, 2.0 ** -8)
        counts += ref["counts"]
    want_b = mo.bias_update(b, counts, w.K, W * w.T, 0.01)
    assert np.array_equal(bd.cpu().numpy().view(np.int32), want_b.view(np.int32))
    assert np.float32(mv.item()) == np.float32(mo.max_vio(counts, w.K, W * w.T, w.E_r))

"""moe_permute_noalloc: the workspace-free dispatch variant for callers that
cannot allocate device memory (their memory all belongs to their own pool,
they enqueue while another thread captures a CUDA graph, or they cannot accept
cudaMalloc's implicit synchronisation).  Through the C ABI, two calls in a row
must give exactly what moe_permute gives with a workspace -- dispatch is
integer work, so the tolerance of the other dispatch tests applies: bit-exact.
The second call uses other inputs, so a histogram left over from the first
call would show.  Collected last on purpose (file name)."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as mo
import sparse_mixture_experts_selection_b200 as moe

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


def _case(T, E, K, d, cf, seed):
    rng = np.random.default_rng(seed)
    z = rng.normal(size=(T, E)).astype(np.float32) + np.linspace(0, 1.5, E, dtype=np.float32)
    s = mo.sigmoid_scores(z)
    idx = mo.select_experts(s, np.zeros(E, np.float32), K)
    gates = mo.gates_from_scores(s, idx)
    h = rng.normal(size=(T, d)).astype(np.float32)
    cfg = moe.MoeConfig(T=T, d_model=d, E_r=E, E_s=0, K=K, d_ffn=64, d_ffn_shared=0, score_fn=0,
                        n_groups=1, topk_groups=1, group_topn=0, capacity_factor=cf, dtype=1,
                        add_residual=1)
    dev = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)
    return cfg, dev(idx, torch.int32), dev(gates), dev(h, torch.bfloat16)


def _outputs(cfg):
    T, K, E, d = cfg.T, cfg.K, cfg.E_r, cfg.d_model
    i32 = lambda *s: torch.full(s, -5, dtype=torch.int32, device="cuda")
    return dict(offsets=i32(E + 1), perm_tok=i32(T * K), row_of=i32(T, K), kept=i32(E),
                row_gate=torch.zeros(T * K, dtype=torch.float32, device="cuda"),
                x_perm=torch.zeros((T * K, d), dtype=torch.bfloat16, device="cuda"))


def _with_workspace(cfg, idx, gates, h):
    o = _outputs(cfg)
    ws = moe.alloc_workspace(moe.moe_workspace_size(cfg))
    moe.moe_permute(cfg, idx, gates, h, o["offsets"], o["perm_tok"], o["row_of"], o["kept"],
                    o["row_gate"], o["x_perm"], ws)
    return o


def _without_workspace(cfg, idx, gates, h):
    o = _outputs(cfg)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_permute_noalloc(cfg, idx, gates, h, o["offsets"], o["perm_tok"], o["row_of"], o["kept"],
                            o["row_gate"], o["x_perm"], err)
    o["err"] = err
    return o


def test_noalloc_permute_matches_workspace_permute_twice():
    for T, E, K, d, cf, seed in [(1500, 64, 8, 128, 0.0, 1), (700, 32, 4, 64, 1.25, 2)]:
        cfg, idx, gates, h = _case(T, E, K, d, cf, seed)
        want = _with_workspace(cfg, idx, gates, h)
        got = _without_workspace(cfg, idx, gates, h)
        torch.cuda.synchronize()
        assert got["err"].item() == 0
        n = int(want["offsets"][-1].item())
        for k in ("offsets", "kept", "row_of"):
            assert torch.equal(got[k], want[k]), k
        assert torch.equal(got["perm_tok"][:n], want["perm_tok"][:n])
        assert torch.equal(got["row_gate"][:n], want["row_gate"][:n])
        assert torch.equal(got["x_perm"][:n].view(torch.int16), want["x_perm"][:n].view(torch.int16))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    cfg, idx, gates, h = _case(64, 8, 2, 64, 0.0, 3)
    cfg.T, cfg.E_r = 1 << 20, 1024          # 2 * 4096 * 1024 words > the fixed array
    with pytest.raises(moe.MoeError) as exc:
        moe.moe_permute_noalloc(cfg, idx, gates, None, idx, idx, idx, idx, None, None)
    assert exc.value.status == 2

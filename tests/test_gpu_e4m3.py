"""e4m3 expert weights on the GPU against the oracle: the row quantizer bit for
bit (codes and power-of-two scales), the expert FFN entry point and the whole
layer (e4m3 x e4m3 tensor-core GEMMs with fp32 accumulation) within the bf16
output bar.

Both sides quantize the same values with the same rule, and a power-of-two
scale makes x / s exact, so the codes agree exactly; what remains is the
accumulation order of the GEMMs (fp32 on the tensor cores, float64 in the
oracle) and the bf16 storage of A and of the outputs."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as mo
import sparse_mixture_experts_selection_b200 as moe
from gpu_helpers import BF16_TOL, HostWeights, Layer, check_close, oracle_cfg, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

W = mi.WORKLOADS
SMALL_E4M3 = {
    "deepseek_small_e4m3": W["deepseek_v3_e4m3"].with_(T=520, d_model=256, E_r=64, E_s=1, K=6, d_ffn=256,
                                                       d_ffn_shared=384, n_groups=8, topk_groups=3),
    "finegrained_near_tile_e4m3": W["finegrained_64x1408"].with_(
        T=440, d_model=192, E_r=16, E_s=2, K=4, d_ffn=192, d_ffn_shared=144, dtype="bf16_e4m3"),
    "mixtral_small_e4m3": W["mixtral_8x14336"].with_(T=300, d_model=256, d_ffn=320, dtype="bf16_e4m3"),
    # capacity 1.0: 99 of the 1760 (token, expert) pairs are dropped
    "finegrained_cf_e4m3": W["finegrained_64x1408"].with_(
        T=440, d_model=192, E_r=16, E_s=2, K=4, d_ffn=192, d_ffn_shared=128, capacity_factor=1.0,
        dtype="bf16_e4m3"),
    "decode_small_e4m3": W["deepseek_v3_decode_e4m3"].with_(T=24, d_model=320, E_r=64, d_ffn=128,
                                                            d_ffn_shared=128, topk_groups=4),
}


def quantize_gpu(x: np.ndarray, src_dtype: int):
    n, c = x.shape
    src = to_dev(x, torch.bfloat16 if src_dtype == moe.DTYPE_BF16 else torch.float32)
    dst = torch.full((moe.moe_quantized_bytes(n, c),), 0x55, dtype=torch.uint8, device="cuda")
    moe.moe_quantize_rows(src, src_dtype, n, c, dst)
    torch.cuda.synchronize()
    out = dst.cpu().numpy()
    return out[: n * c].reshape(n, c), out[n * c:].view(np.float32)


@pytest.mark.parametrize("src_dtype", [moe.DTYPE_BF16, moe.DTYPE_F32])
@pytest.mark.parametrize("shape", [(1, 16), (37, 48), (300, 7168), (64, 2048)])
def test_quantize_rows_bit_exact(src_dtype, shape):
    n, c = shape
    rng = np.random.default_rng(n * 31 + c)
    x = (rng.normal(size=(n, c)) * rng.choice([1e-30, 1e-3, 1.0, 600.0, 3e20], size=(n, 1))).astype(np.float32)
    x[0, : min(c, 8)] = [-1e-38, 0.0, -0.0, 448.0, -448.0, 1e-5, 7.0, -3.5][: min(c, 8)]
    if n > 2:
        x[2] = 0.0                                     # all-zero row: scale 1, codes 0
    if src_dtype == moe.DTYPE_BF16:
        x = mi.round_bf16(x)
    codes, scales = quantize_gpu(x, src_dtype)
    want_c, want_s = mo.quantize_rows(x)
    assert np.array_equal(scales.view(np.int32), want_s.view(np.int32))
    assert np.array_equal(codes, want_c)


def test_expert_ffn_entry_e4m3():
    n_exp, d, f = 5, 192, 208
    rows = np.array([0, 130, 0, 257, 1], dtype=np.int64)
    offsets = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    R = int(offsets[-1])
    rng = np.random.default_rng(3)
    rnd = lambda *s, sc=1.0: mi.round_bf16((rng.normal(size=s) * sc).astype(np.float32))
    x, wg, wu = rnd(R, d), rnd(n_exp, f, d, sc=d ** -0.5), rnd(n_exp, f, d, sc=d ** -0.5)
    wd, scale = rnd(n_exp, d, f, sc=f ** -0.5), rng.uniform(0.1, 1, size=R).astype(np.float32)
    cfg = moe.MoeConfig(T=R, d_model=d, E_r=n_exp, E_s=0, K=1, d_ffn=f, d_ffn_shared=0, score_fn=0,
                        n_groups=1, topk_groups=1, group_topn=0, capacity_factor=0.0,
                        dtype=moe.DTYPE_BF16_E4M3, add_residual=1)

    def blob(wt):
        n, r, c = wt.shape
        q = torch.empty(moe.moe_quantized_bytes(n * r, c), dtype=torch.uint8, device="cuda")
        moe.moe_quantize_rows(to_dev(wt, torch.bfloat16), moe.DTYPE_BF16, n * r, c, q)
        return q

    max_rows = R + 3
    ws = moe.alloc_workspace(moe.moe_expert_ffn_workspace_size(cfg, n_exp, f, max_rows))
    xd = torch.zeros((max_rows, d), dtype=torch.bfloat16, device="cuda")
    xd[:R] = to_dev(x, torch.bfloat16)
    out = torch.full((max_rows, d), 7.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(cfg, n_exp, f, max_rows, to_dev(offsets, torch.int32), xd, blob(wg), blob(wu),
                       blob(wd), to_dev(scale), out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    got = out.float().cpu().numpy()
    want = np.zeros((R, d))
    for g in range(n_exp):
        a, b_ = offsets[g], offsets[g + 1]
        if b_ > a:
            want[a:b_] = scale[a:b_, None] * mo.swiglu_q8(x[a:b_], mo.quantize_rows(wg[g]),
                                                          mo.quantize_rows(wu[g]), mo.quantize_rows(wd[g]))
    err = np.max(np.abs(got[:R] - want) - 2.0 ** -8 * np.abs(want))
    assert err <= BF16_TOL * np.sqrt(np.mean(want ** 2)), err
    assert np.all(got[R:] == 7.0)


def device_blobs(HW):
    out = {}
    for k in ("gate", "up", "down", "sgate", "sup", "sdown"):
        a = HW.arrays.get(k)
        if a is None:
            out[k] = None
            continue
        n, r, c = a.shape
        q = torch.empty(moe.moe_quantized_bytes(n * r, c), dtype=torch.uint8, device="cuda")
        moe.moe_quantize_rows(to_dev(a, torch.bfloat16), moe.DTYPE_BF16, n * r, c, q)
        out[k] = q
    return out


def q8_source(HW):
    cache = {}

    def get(which, ex):
        key = (which, int(ex))
        if key not in cache:
            cache[key] = mo.quantize_rows(HW.arrays[which][ex])
        return cache[key]
    return get


@pytest.mark.parametrize("name", sorted(SMALL_E4M3))
def test_layer_e4m3_fed_scores(name):
    w = SMALL_E4M3[name]
    h, e, b = mi.gen_h(w, 0), mi.gen_centroids(w), mi.gen_bias(w)
    HW = HostWeights(w)
    cfg = oracle_cfg(w)
    s = mo.affinity(h, e, w.score_fn)
    b_sel = b if w.score_fn == 0 else np.zeros(w.E_r, np.float32)
    idx, gates, disp = mo.route(cfg, s, b_sel)
    want = mo.layer_output_q8(cfg, h, idx, gates, disp, q8_source(HW))
    L = Layer(w, device_blobs(HW))
    y = L.forward(to_dev(h, torch.bfloat16), None, to_dev(b), s_in=to_dev(s))
    assert L.device_error() == 0
    assert np.array_equal(L.idx.cpu().numpy(), idx)
    assert np.array_equal(L.kept.cpu().numpy(), disp.kept)
    check_close(y.float().cpu().numpy(), want, h, BF16_TOL, bool(w.add_residual), 2.0 ** -8)


def test_layer_e4m3_independent_routing():
    w = SMALL_E4M3["deepseek_small_e4m3"]
    h, e, b = mi.gen_h(w, 0), mi.gen_centroids(w), mi.gen_bias(w)
    HW = HostWeights(w)
    cfg = oracle_cfg(w)
    s = mo.affinity(h, e, w.score_fn)
    idx, gates, disp = mo.route(cfg, s, b)
    want = mo.layer_output_q8(cfg, h, idx, gates, disp, q8_source(HW))
    L = Layer(w, device_blobs(HW))
    y = L.forward(to_dev(h, torch.bfloat16), to_dev(e), to_dev(b)).float().cpu().numpy()
    assert L.device_error() == 0
    fragile = mo.near_tie_tokens(s, b, w.K, w.n_groups, w.topk_groups, w.group_topn, 1e-5)
    same = np.all(L.idx.cpu().numpy() == idx, axis=1)
    assert np.all(same | fragile)
    check_close(y[same], want[same], h[same], BF16_TOL, True, 2.0 ** -8)


def test_e4m3_layer_tracks_the_bf16_layer():
    """The quantized layer's expert contribution stays within 10 % (RMS) of the
    bf16 layer's (the format's own error, ~6 % for three roundings to 3
    mantissa bits)."""
    w = SMALL_E4M3["deepseek_small_e4m3"]
    h, e, b = mi.gen_h(w, 0), mi.gen_centroids(w), mi.gen_bias(w)
    HW = HostWeights(w)
    s = to_dev(mo.affinity(h, e, w.score_fn))
    hd, bd = to_dev(h, torch.bfloat16), to_dev(b)
    Lq = Layer(w, device_blobs(HW))
    yq = Lq.forward(hd, None, bd, s_in=s).float().cpu().numpy()
    Lb = Layer(w.with_(dtype="bf16"), HW.device())
    yb = Lb.forward(hd, None, bd, s_in=s).float().cpu().numpy()
    dq, db = yq - h, yb - h
    rel = np.sqrt(np.mean((dq - db) ** 2)) / np.sqrt(np.mean(db ** 2))
    assert 1e-3 < rel < 0.10, rel

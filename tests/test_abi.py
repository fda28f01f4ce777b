"""The C-ABI library loads, exports every symbol include/moe.h declares, and
validates its arguments on the host (no GPU needed: every call below fails
validation before any CUDA call is made)."""
import ctypes
import os
import re

import pytest

import moe_inputs as mi
import sparse_mixture_experts_selection_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 1 << 20       # an aligned, never-dereferenced stand-in for a device pointer


def header_symbols():
    txt = open(os.path.join(ROOT, "include", "moe.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    L = moe.lib()
    syms = header_symbols()
    assert len(syms) >= 12
    for s in syms:
        assert hasattr(L, s), s
    assert set(syms) == set(moe.SIGNATURES), set(syms) ^ set(moe.SIGNATURES)
    assert L.moe_abi_version() == 4
    assert moe.lib().moe_status_string(3) == b"MOE_ERR_WORKSPACE"


def cfg_of(name, **kw):
    return moe.config_for(mi.WORKLOADS[name], **kw)


@pytest.mark.parametrize("name", sorted(mi.WORKLOADS))
def test_workspace_size_of_every_workload(name):
    w = mi.WORKLOADS[name]
    n = moe.moe_workspace_size(cfg_of(name))
    es = 2 if w.dtype != "f32" else 4
    # at least: permuted rows + their SwiGLU products + gate-scaled slots
    R = min(w.T * w.K, w.E_r * (mi_capacity(w)))
    assert n >= R * (2 * w.d_model + w.d_ffn) * es
    assert n < 64 * 1024 ** 3


def mi_capacity(w):
    from oracle import moe_oracle as mo
    return mo.capacity(w.T, w.K, w.E_r, w.capacity_factor)


@pytest.mark.parametrize("field,value,status", [
    ("K", 0, 1), ("K", 9, 1), ("T", 0, 1), ("d_model", 12, 1), ("E_r", 0, 1),
    ("E_r", 2048, 2), ("E_s", -1, 1), ("E_s", 9, 2), ("score_fn", 2, 1), ("dtype", 3, 1),
    ("d_ffn", 4, 1), ("n_groups", 0, 1), ("add_residual", 2, 1),
])
def test_invalid_config_rejected(field, value, status):
    c = cfg_of("toy_fp32", **{field: value})
    n = ctypes.c_size_t(0)
    st = moe.lib().moe_workspace_size(ctypes.byref(c), ctypes.byref(n))
    assert st == status, moe.lib().moe_last_error_detail()


def test_group_constraints():
    L = moe.lib()
    n = ctypes.c_size_t(0)
    ok = cfg_of("deepseek_v3")
    assert L.moe_workspace_size(ctypes.byref(ok), ctypes.byref(n)) == 0
    for kw, st in [(dict(n_groups=7), 1), (dict(topk_groups=0), 1), (dict(topk_groups=9), 1),
                   (dict(group_topn=33), 1), (dict(n_groups=256, topk_groups=1, K=1), 1),
                   (dict(n_groups=64, topk_groups=1, K=4), 2)]:
        c = cfg_of("deepseek_v3", **kw)
        assert L.moe_workspace_size(ctypes.byref(c), ctypes.byref(n)) == st, (kw, L.moe_last_error_detail())
    # topk_groups * group size < K
    c = cfg_of("deepseek_v3", topk_groups=1, K=33)
    assert L.moe_workspace_size(ctypes.byref(c), ctypes.byref(n)) in (1, 2)


def test_expert_ffn_tile_rows_validation_and_fp32():
    """The tile query validates on the host; an fp32 layer answers with the
    CUDA-core tile without touching the device."""
    L = moe.lib()
    c = cfg_of("toy_fp32")
    n = ctypes.c_int32(-1)
    assert L.moe_expert_ffn_tile_rows(ctypes.byref(c), 8, 1024, None) == 1
    assert L.moe_expert_ffn_tile_rows(ctypes.byref(c), 0, 1024, ctypes.byref(n)) == 1
    assert L.moe_expert_ffn_tile_rows(ctypes.byref(c), 8, -1, ctypes.byref(n)) == 1
    assert moe.moe_expert_ffn_tile_rows(c, 8, 4096) == 32


def test_bf16_small_dims_unsupported():
    c = cfg_of("toy_fp32", dtype=moe.DTYPE_BF16, d_model=32)
    n = ctypes.c_size_t(0)
    assert moe.lib().moe_workspace_size(ctypes.byref(c), ctypes.byref(n)) == 2


def test_entry_points_validate_pointers_before_any_launch():
    L = moe.lib()
    c = cfg_of("toy_fp32")
    need = moe.moe_workspace_size(c)
    P = FAKE
    # NULL inputs
    assert L.moe_layer_forward(ctypes.byref(c), None, P, P, P, P, P, None, None, None, None, P,
                               None, None, None, None, None, None, 0, 0.0, None, P, need, None) == 1
    # too small / misaligned workspace
    assert L.moe_layer_forward(ctypes.byref(c), P, P, P, P, P, P, None, None, None, None, P,
                               None, None, None, None, None, None, 0, 0.0, None, P, need - 1, None) == 3
    assert L.moe_layer_forward(ctypes.byref(c), P, P, P, P, P, P, None, None, None, None, P,
                               None, None, None, None, None, None, 0, 0.0, None, P + 16, need, None) == 3
    # misaligned activation pointer
    assert L.moe_layer_forward(ctypes.byref(c), P + 4, P, P, P, P, P, None, None, None, None, P,
                               None, None, None, None, None, None, 0, 0.0, None, P, need, None) == 1
    # update_bias without b, non-finite gamma
    assert L.moe_layer_forward(ctypes.byref(c), P, P, None, P, P, P, None, None, None, None, P,
                               None, None, None, None, None, None, 1, 0.1, None, P, need, None) == 1
    assert L.moe_layer_forward(ctypes.byref(c), P, P, P, P, P, P, None, None, None, None, P,
                               None, None, None, None, None, None, 1, float("nan"), None, P, need, None) == 1
    # shared experts configured but their weights missing
    c2 = cfg_of("finegrained_64x1408")
    n2 = moe.moe_workspace_size(c2)
    assert L.moe_layer_forward(ctypes.byref(c2), P, P, P, P, P, P, None, None, None, None, P,
                               None, None, None, None, None, None, 0, 0.0, None, P, n2, None) == 1
    # route: idx/gates required; permute: row_gate needs gates
    assert L.moe_route(ctypes.byref(c), P, P, None, None, None, None, None, P, None, P, need, None) == 1
    assert L.moe_permute(ctypes.byref(c), P, None, None, P, P, P, P, P, None, P, need, None) == 1
    assert L.moe_bias_update(ctypes.byref(c), None, 0.1, P, None, None) == 1
    assert L.moe_combine(ctypes.byref(c), P, None, None, P, P, None) == 1
    assert b"NULL" in L.moe_last_error_detail()
    # expert FFN workspace query and its own validation
    n = ctypes.c_size_t(0)
    assert L.moe_expert_ffn_workspace_size(ctypes.byref(c), 0, 128, 10, ctypes.byref(n)) == 1
    assert L.moe_expert_ffn_workspace_size(ctypes.byref(c), 8, 128, 10, ctypes.byref(n)) == 0
    assert L.moe_expert_ffn(ctypes.byref(c), 8, 128, 10, P, P, P, P, P, None, P, P, n.value - 1, None) == 3
    assert L.moe_get_device_error(None, None) == 1
    # expert-parallel plan: world, rank and the expert split are checked before any launch
    assert L.moe_ep_plan(P, 0, 0, 16, 10, P, P, P, P, None, None) == 1          # world < 1
    assert L.moe_ep_plan(P, 65, 0, 65 * 4, 10, P, P, P, P, None, None) == 1     # world > 64
    assert L.moe_ep_plan(P, 4, 4, 16, 10, P, P, P, P, None, None) == 1          # rank >= world
    assert L.moe_ep_plan(P, 3, 0, 16, 10, P, P, P, P, None, None) == 1          # E_r % world
    assert L.moe_ep_plan(P, 4, 0, 2048, 10, P, P, P, P, None, None) == 1        # E_r > 1024
    assert L.moe_ep_plan(P, 4, 0, 16, -1, P, P, P, P, None, None) == 1          # max_recv < 0
    assert L.moe_ep_plan(P, 4, 0, 16, 10, P, P, None, P, None, None) == 1       # regroup NULL
    assert L.moe_ep_plan(P + 2, 4, 0, 16, 10, P, P, P, P, None, None) == 1      # misaligned offsets
    # router statistics: seq_len must divide T; stats required
    n = ctypes.c_size_t(0)
    assert L.moe_router_stats_workspace_size(ctypes.byref(c), 7, ctypes.byref(n)) == 1
    assert L.moe_router_stats_workspace_size(ctypes.byref(c), 128, ctypes.byref(n)) == 0
    assert L.moe_router_stats(ctypes.byref(c), P, None, P, None, 128, 0.01, 1e-3, 1e-4, None, P,
                              n.value, None) == 1

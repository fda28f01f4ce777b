"""B200 (sm_100a) forward pass of one sparse Mixture-of-Experts layer.

Thin Python binding of the C ABI in include/moe.h (libmoe.so): argument
marshalling only.  Every step of the layer runs in the library's CUDA kernels;
there is no CPU or PyTorch fallback -- importing this package fails loudly when
the library is missing or does not load.

PyTorch provides the device memory and the stream: tensors are passed by
pointer (``tensor.data_ptr()``) and work is enqueued on
``torch.cuda.current_stream()`` unless a stream is given.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

from ._build import LIB_PATH

__all__ = [
    "MoeConfig", "MoeError", "lib", "config_for", "moe_workspace_size", "moe_route", "moe_permute",
    "moe_expert_ffn", "moe_expert_ffn_workspace_size", "moe_combine", "moe_bias_update",
    "moe_layer_forward", "moe_get_device_error", "moe_clear_device_error", "alloc_workspace",
    "moe_router_stats", "moe_router_stats_workspace_size", "ROUTER_STATS", "moe_permute_noalloc",
    "moe_quantized_bytes", "moe_quantize_rows", "DTYPE_BF16_E4M3", "moe_layer_backward", "moe_gather_rows",
    "moe_set_phase_events", "moe_selftest_bounded_wait", "moe_ep_plan", "moe_expert_ffn_tile_rows",
    "SCORE_SIGMOID", "SCORE_SOFTMAX", "DTYPE_F32", "DTYPE_BF16",
]

SCORE_SIGMOID, SCORE_SOFTMAX = 0, 1
DTYPE_F32, DTYPE_BF16, DTYPE_BF16_E4M3 = 0, 1, 2
DEVERR_NONE, DEVERR_WAIT_TIMEOUT, DEVERR_INDEX, DEVERR_RANGE = 0, 1, 2, 3
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE"}


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("E_r", ctypes.c_int32),
                ("E_s", ctypes.c_int32), ("K", ctypes.c_int32), ("d_ffn", ctypes.c_int32),
                ("d_ffn_shared", ctypes.c_int32), ("score_fn", ctypes.c_int32),
                ("n_groups", ctypes.c_int32), ("topk_groups", ctypes.c_int32),
                ("group_topn", ctypes.c_int32), ("capacity_factor", ctypes.c_float),
                ("dtype", ctypes.c_int32), ("add_residual", ctypes.c_int32),
                ("train", ctypes.c_int32)]


class MoeError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status


_lib = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32

# (name, restype, argtypes) of every exported symbol of include/moe.h
SIGNATURES = {
    "moe_abi_version": (ctypes.c_int32, []),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_last_error_detail": (ctypes.c_char_p, []),
    "moe_workspace_size": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_expert_ffn_workspace_size": (ctypes.c_int, [_P, _I32, _I32, _I32, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_expert_ffn_tile_rows": (ctypes.c_int, [_P, _I32, _I32, ctypes.POINTER(ctypes.c_int32)]),
    "moe_route": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_permute": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_expert_ffn": (ctypes.c_int, [_P, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P,
                                      ctypes.c_size_t, _P]),
    "moe_combine": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P]),
    "moe_bias_update": (ctypes.c_int, [_P, _P, ctypes.c_float, _P, _P, _P]),
    "moe_layer_forward": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                         _P, _P, _P, _P, _I32, ctypes.c_float, _P, _P,
                                         ctypes.c_size_t, _P]),
    "moe_router_stats_workspace_size": (ctypes.c_int, [_P, _I32, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_quantized_bytes": (ctypes.c_int, [ctypes.c_int64, _I32, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_layer_backward": (ctypes.c_int, [_P] * 20 + [_P, ctypes.c_size_t, _P]),
    "moe_quantize_rows": (ctypes.c_int, [_P, _I32, ctypes.c_int64, _I32, _P, _P]),
    "moe_gather_rows": (ctypes.c_int, [_P, ctypes.c_int64, _I32, _P, ctypes.c_int64, _P, _P]),
    "moe_ep_plan": (ctypes.c_int, [_P, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P]),
    "moe_router_stats": (ctypes.c_int, [_P, _P, _P, _P, _P, _I32, ctypes.c_float, ctypes.c_float,
                                        ctypes.c_float, _P, _P, ctypes.c_size_t, _P]),
    "moe_get_device_error": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int32)]),
    "moe_clear_device_error": (ctypes.c_int, [_P, _P]),
    "moe_set_phase_events": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), _I32]),
    "moe_permute_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_selftest_bounded_wait": (ctypes.c_int, [_P, ctypes.c_int64, _P]),
}

# phases of moe_layer_forward marked by moe_set_phase_events (between marks i and i+1)
PHASES = ["route", "dispatch", "ffn_groups", "ffn_gate_up", "ffn_down", "combine", "bias_step"]


def lib() -> ctypes.CDLL:
    """The loaded libmoe.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m sparse_mixture_experts_selection_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int) -> None:
    if status != 0:
        raise MoeError(status, lib().moe_last_error_detail().decode())


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def config_for(w, **overrides) -> MoeConfig:
    """MoeConfig of a ``moe_inputs.Workload`` (or any object with the same fields)."""
    c = MoeConfig(T=w.T, d_model=w.d_model, E_r=w.E_r, E_s=w.E_s, K=w.K, d_ffn=w.d_ffn,
                  d_ffn_shared=w.d_ffn_shared, score_fn=w.score_fn, n_groups=w.n_groups,
                  topk_groups=w.topk_groups, group_topn=w.group_topn,
                  capacity_factor=w.capacity_factor,
                  dtype={"bf16": DTYPE_BF16, "bf16_e4m3": DTYPE_BF16_E4M3}.get(w.dtype, DTYPE_F32),
                  add_residual=w.add_residual)
    for k, v in overrides.items():
        setattr(c, k, v)
    return c


def moe_workspace_size(cfg: MoeConfig) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def moe_expert_ffn_workspace_size(cfg: MoeConfig, n_experts: int, d_ffn: int, max_rows: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_expert_ffn_workspace_size(ctypes.byref(cfg), n_experts, d_ffn, max_rows, ctypes.byref(n)))
    return n.value


def moe_expert_ffn_tile_rows(cfg: MoeConfig, n_experts: int, max_rows: int) -> int:
    """Row-tile height of the GEMMs moe_expert_ffn runs for these arguments:
    256 on CTA pairs, 128 single-CTA tensor-core, the CUDA-core tile for fp32."""
    n = ctypes.c_int32(0)
    _check(lib().moe_expert_ffn_tile_rows(ctypes.byref(cfg), n_experts, max_rows, ctypes.byref(n)))
    return n.value


def alloc_workspace(nbytes: int, device="cuda"):
    """A zeroed uint8 device tensor usable as a workspace (torch allocations are
    at least 256-byte aligned)."""
    import torch
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def moe_route(cfg, h, e, b, s_in, s_out, idx, gates, counts, ws, stream=None, z_out=None):
    _check(lib().moe_route(ctypes.byref(cfg), _ptr(h), _ptr(e), _ptr(b), _ptr(s_in), _ptr(s_out),
                           _ptr(z_out), _ptr(idx), _ptr(gates), _ptr(counts), _ptr(ws), ws.numel(),
                           _stream(stream)))


def moe_router_stats_workspace_size(cfg: MoeConfig, seq_len: int = 0) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_router_stats_workspace_size(ctypes.byref(cfg), int(seq_len), ctypes.byref(n)))
    return n.value


def moe_gather_rows(src, n_src: int, row_bytes: int, map_, n_rows: int, dst, stream=None):
    """dst[r] = src[map_[r]] row by row (zero where map_[r] < 0)."""
    _check(lib().moe_gather_rows(_ptr(src), int(n_src), int(row_bytes), _ptr(map_), int(n_rows), _ptr(dst),
                                 _stream(stream)))


def moe_quantized_bytes(n_rows: int, cols: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_quantized_bytes(int(n_rows), int(cols), ctypes.byref(n)))
    return n.value


def moe_quantize_rows(src, src_dtype: int, n_rows: int, cols: int, dst, stream=None):
    _check(lib().moe_quantize_rows(_ptr(src), int(src_dtype), int(n_rows), int(cols), _ptr(dst),
                                   _stream(stream)))


def moe_layer_backward(cfg, h, e, s, idx, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, dy, dh, de,
                       dw_gate, dw_up, dw_down, dws_gate, dws_up, dws_down, ws, stream=None):
    """Gradients of the last moe_layer_forward (cfg.train = 1, same workspace)."""
    _check(lib().moe_layer_backward(
        ctypes.byref(cfg), _ptr(h), _ptr(e), _ptr(s), _ptr(idx), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
        _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(dy), _ptr(dh), _ptr(de), _ptr(dw_gate), _ptr(dw_up),
        _ptr(dw_down), _ptr(dws_gate), _ptr(dws_up), _ptr(dws_down), _ptr(ws), ws.numel(), _stream(stream)))


# order of the values moe_router_stats writes
ROUTER_STATS = ["aux_loss", "z_loss", "seq_balance_loss", "load_entropy", "max_vio", "dropped_rate"]


def moe_router_stats(cfg, s, z, idx, kept, stats, ws, seq_len=0, alpha_aux=0.01, c_z=1e-3,
                     alpha_seq=1e-4, stream=None):
    _check(lib().moe_router_stats(ctypes.byref(cfg), _ptr(s), _ptr(z), _ptr(idx), _ptr(kept),
                                  int(seq_len), float(alpha_aux), float(c_z), float(alpha_seq),
                                  _ptr(stats), _ptr(ws), ws.numel(), _stream(stream)))


def moe_permute(cfg, idx, gates, h, offsets, perm_tok, row_of, kept, row_gate, x_perm, ws, stream=None):
    _check(lib().moe_permute(ctypes.byref(cfg), _ptr(idx), _ptr(gates), _ptr(h), _ptr(offsets),
                             _ptr(perm_tok), _ptr(row_of), _ptr(kept), _ptr(row_gate), _ptr(x_perm),
                             _ptr(ws), ws.numel(), _stream(stream)))


def moe_permute_noalloc(cfg, idx, gates, h, offsets, perm_tok, row_of, kept, row_gate, x_perm,
                        dev_error=None, stream=None):
    """moe_permute with no workspace: for callers that cannot allocate device
    memory (see include/moe.h); scratch is a fixed array inside the library."""
    _check(lib().moe_permute_noalloc(ctypes.byref(cfg), _ptr(idx), _ptr(gates), _ptr(h), _ptr(offsets),
                                     _ptr(perm_tok), _ptr(row_of), _ptr(kept), _ptr(row_gate),
                                     _ptr(x_perm), _ptr(dev_error), _stream(stream)))


def moe_ep_plan(offsets_all, world, rank, E_r, max_recv, splits, local_offsets, regroup, inverse,
                dev_error=None, stream=None):
    """Exchange plan of an expert-parallel layer on the device (see include/moe.h)."""
    _check(lib().moe_ep_plan(_ptr(offsets_all), world, rank, E_r, max_recv, _ptr(splits), _ptr(local_offsets),
                             _ptr(regroup), _ptr(inverse), _ptr(dev_error), _stream(stream)))


def moe_expert_ffn(cfg, n_experts, d_ffn, max_rows, offsets, x, w_gate, w_up, w_down, row_scale,
                   out, ws, stream=None):
    _check(lib().moe_expert_ffn(ctypes.byref(cfg), n_experts, d_ffn, max_rows, _ptr(offsets), _ptr(x),
                                _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(row_scale), _ptr(out),
                                _ptr(ws), ws.numel(), _stream(stream)))


def moe_combine(cfg, h, slot, shared_out, row_of, y, stream=None):
    _check(lib().moe_combine(ctypes.byref(cfg), _ptr(h), _ptr(slot), _ptr(shared_out), _ptr(row_of),
                             _ptr(y), _stream(stream)))


def moe_bias_update(cfg, counts, gamma, b, max_vio, stream=None):
    _check(lib().moe_bias_update(ctypes.byref(cfg), _ptr(counts), float(gamma), _ptr(b), _ptr(max_vio),
                                 _stream(stream)))


def moe_layer_forward(cfg, h, e, b, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, y, ws, *,
                      s_in=None, idx_out=None, gates_out=None, counts_out=None, kept_out=None,
                      s_out=None, z_out=None, update_bias=False, gamma=0.0, max_vio_out=None,
                      stream=None):
    _check(lib().moe_layer_forward(
        ctypes.byref(cfg), _ptr(h), _ptr(e), _ptr(b), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
        _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(s_in), _ptr(y), _ptr(idx_out), _ptr(gates_out),
        _ptr(counts_out), _ptr(kept_out), _ptr(s_out), _ptr(z_out), int(bool(update_bias)), float(gamma),
        _ptr(max_vio_out), _ptr(ws), ws.numel(), _stream(stream)))


def moe_get_device_error(ws) -> int:
    code = ctypes.c_int32(0)
    st = lib().moe_get_device_error(_ptr(ws), ctypes.byref(code))
    if st not in (0, 5):
        _check(st)
    return code.value


def moe_set_phase_events(events) -> None:
    """Record these torch.cuda.Event objects (up to 8) at the phase boundaries of
    every later moe_layer_forward call in this thread; [] turns it off."""
    arr = (ctypes.c_void_p * max(1, len(events)))(*[ev.cuda_event for ev in events])
    _check(lib().moe_set_phase_events(arr, len(events)))


def moe_selftest_bounded_wait(ws, limit_ns: int = 50_000_000, stream=None) -> None:
    """Enqueue the failure-detection self-test (see include/moe.h)."""
    _check(lib().moe_selftest_bounded_wait(_ptr(ws), int(limit_ns), _stream(stream)))


def moe_clear_device_error(ws, stream=None) -> None:
    _check(lib().moe_clear_device_error(_ptr(ws), _stream(stream)))

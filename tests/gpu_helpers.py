"""Helpers shared by the GPU parity tests: device copies of the generator's
inputs, one call of the layer through the C ABI, and the tolerance checks.

Every input comes from moe_inputs (numpy, or its bit-identical C/CUDA twins);
every expected value comes from oracle/.  Nothing the CUDA library computes is
ever fed to the oracle.
"""
from __future__ import annotations

import functools

import numpy as np
import torch

import moe_inputs as mi
from moe_inputs import native
from oracle import moe_oracle as mo
import sparse_mixture_experts_selection_b200 as moe

BF16_TOL = 2e-2   # max |y - y_ref| <= BF16_TOL * RMS (bf16 layers)
F32_TOL = 1e-4    # ... for fp32 layers


def torch_dtype(w):
    return torch.bfloat16 if w.dtype != "f32" else torch.float32


def to_dev(x: np.ndarray, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device="cuda", dtype=dtype)


def oracle_cfg(w) -> mo.LayerConfig:
    return mo.LayerConfig(T=w.T, d_model=w.d_model, E_r=w.E_r, E_s=w.E_s, K=w.K,
                          score_fn=w.score_fn, n_groups=w.n_groups, topk_groups=w.topk_groups,
                          group_topn=w.group_topn, capacity_factor=w.capacity_factor,
                          add_residual=w.add_residual)


class HostWeights:
    """Numpy weights of a small workload (all experts in memory)."""

    def __init__(self, w):
        self.w = w
        self.arrays = {k: mi.gen_weight(w, k) for k in ("gate", "up", "down")}
        if w.E_s:
            self.arrays.update({k: mi.gen_weight(w, k) for k in ("sgate", "sup", "sdown")})

    def source(self):
        return lambda which, ex: self.arrays[which][ex]

    def device(self):
        dt = torch_dtype(self.w)
        out = {k: to_dev(v, dt) for k, v in self.arrays.items()}
        for k in ("sgate", "sup", "sdown"):
            out.setdefault(k, None)
        return out


class LazyHostWeights:
    """Per-expert weights regenerated on the host by the C twin of the generator
    (for full-size workloads, where only a few experts are ever needed)."""

    def __init__(self, w):
        self.w = w

    @functools.lru_cache(maxsize=64)
    def get(self, which, ex):
        return native.weight_host(self.w, which, int(ex))

    def source(self):
        return lambda which, ex: self.get(which, int(ex))


def device_weights(w):
    """All weights of a workload generated directly on the device (CUDA twin)."""
    dt = torch_dtype(w)
    bf16 = w.dtype != "f32"
    out = {}
    for k in ("gate", "up", "down", "sgate", "sup", "sdown"):
        tid, n, rows, cols, sigma = mi.weight_spec(w, k)
        if n == 0:
            out[k] = None
            continue
        t = torch.empty((n, rows, cols), dtype=dt, device="cuda")
        native.fill_device(t.data_ptr(), t.numel(), bf16, w.seed, tid, 0, sigma,
                           stream=torch.cuda.current_stream().cuda_stream)
        out[k] = t
    return out


class Layer:
    """Device buffers + workspace for repeated layer calls of one workload."""

    def __init__(self, w, weights):
        self.w = w
        self.cfg = moe.config_for(w)
        self.W = weights
        self.ws = moe.alloc_workspace(moe.moe_workspace_size(self.cfg))
        T, K, E = w.T, w.K, w.E_r
        self.y = torch.empty((T, w.d_model), dtype=torch_dtype(w), device="cuda")
        self.idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
        self.gates = torch.empty((T, K), dtype=torch.float32, device="cuda")
        self.counts = torch.empty(E, dtype=torch.int32, device="cuda")
        self.kept = torch.empty(E, dtype=torch.int32, device="cuda")
        self.s = torch.empty((T, E), dtype=torch.float32, device="cuda")
        self.z = torch.empty((T, E), dtype=torch.float32, device="cuda")
        self.max_vio = torch.empty(1, dtype=torch.float32, device="cuda")

    def forward(self, h, e, b, s_in=None, update_bias=False, gamma=0.0):
        W = self.W
        moe.moe_layer_forward(self.cfg, h, e, b, W["gate"], W["up"], W["down"], W["sgate"], W["sup"],
                              W["sdown"], self.y, self.ws, s_in=s_in, idx_out=self.idx,
                              gates_out=self.gates, counts_out=self.counts, kept_out=self.kept,
                              s_out=self.s, z_out=self.z, update_bias=update_bias, gamma=gamma,
                              max_vio_out=self.max_vio)
        return self.y

    def device_error(self):
        torch.cuda.synchronize()
        return moe.moe_get_device_error(self.ws)


def rms(x: np.ndarray) -> float:
    return float(np.sqrt(np.mean(np.square(np.asarray(x, np.float64)))))


def check_close(y_gpu: np.ndarray, y_ref: np.ndarray, h: np.ndarray, tol: float, residual: bool = True,
                out_eps: float = 2.0 ** -8):
    """The bar: max|y - y_ref| <= tol * RMS(y_ref).  A stricter check keeps the
    residual from hiding expert errors: after allowing for the rounding of the
    stored output (out_eps * |y_ref|, with out_eps = 2^-8 for bf16 and 2^-22
    for fp32: twice the unit roundoff), the error must also stay below
    tol * RMS(y_ref - h).  Returns (err, rms_y, rms_delta)."""
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    assert np.all(np.isfinite(y_gpu)), "non-finite output"
    if not y_ref.size:
        return 0.0, 0.0, 0.0
    diff = np.abs(y_gpu - y_ref)
    err = float(np.max(diff))
    r_y = rms(y_ref)
    r_d = rms(y_ref - (np.asarray(h, np.float64) if residual else 0.0))
    if residual:
        # the layer-output bar (stated for layers with the residual); without the
        # residual y is the bf16-rounded expert sum itself and only the
        # rounding-aware check below applies
        assert err <= tol * r_y, (err, r_y)
    strict = float(np.max(diff - out_eps * np.abs(y_ref)))
    assert strict <= tol * r_d, (strict, r_d)
    return err, r_y, r_d


def out_eps_of(w) -> float:
    return 2.0 ** -8 if w.dtype != "f32" else 2.0 ** -22

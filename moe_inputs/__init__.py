"""Seeded synthetic inputs for the sparse MoE layer: the one module that both the
CUDA path's tests/benchmarks and the CPU oracle draw their inputs from.

It holds no arithmetic of the MoE method itself (no routing, no expert math):
only a counter-based random generator and the recipes that turn its draws into
token activations h, router centroids e, expert biases b and SwiGLU weights.

Generator (counter-based, so any slice of any tensor can be regenerated alone):

* SplitMix64 finaliser ``mix`` (Steele, Lea & Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014) applied to a Weyl sequence:
  draw n of stream (seed, tensor_id) is ``mix(key + (n + 1) * GOLDEN)`` with
  ``key = mix(mix(seed) + tensor_id * GOLDEN)`` (all mod 2**64).
* Normal variates: the four 16-bit fields of one draw are summed (an
  Irwin-Hall sum of four discrete uniforms), centred, and scaled by
  sqrt(3)/65536 so the variance is 1 (to within 2**-32).  Only integer
  arithmetic and one IEEE double multiply are involved, so the CUDA twin in
  ``gen.cu`` reproduces every value bit for bit.  The support is bounded at
  +-3.46 sigma, which is immaterial for these workloads.
* Uniform variates: the top 53 bits of one draw, mapped to [lo, hi) in double.
* Rounding: double -> float32 round-to-nearest-even, then (bf16 tensors)
  float32 -> bf16 round-to-nearest-even.

Element n of a tensor is its row-major flat index, so expert i's slice of a
stacked weight tensor [E, rows, cols] is the contiguous range
[i*rows*cols, (i+1)*rows*cols).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
SQRT3_OVER_65536 = math.sqrt(3.0) / 65536.0
IRWIN_HALL_CENTRE = 131070  # 4 * 32767.5

# tensor ids of one workload's streams (the step index is folded in for h)
TID_H, TID_E, TID_B, TID_WG, TID_WU, TID_WD, TID_WSG, TID_WSU, TID_WSD = range(1, 10)


def _mix_int(x: int) -> int:
    x &= MASK64
    x = ((x ^ (x >> 30)) * _M1) & MASK64
    x = ((x ^ (x >> 27)) * _M2) & MASK64
    return x ^ (x >> 31)


def _mix_np(x: np.ndarray) -> np.ndarray:
    x = x ^ (x >> np.uint64(30))
    x = x * np.uint64(_M1)
    x = x ^ (x >> np.uint64(27))
    x = x * np.uint64(_M2)
    return x ^ (x >> np.uint64(31))


def stream_key(seed: int, tensor_id: int) -> int:
    return _mix_int(_mix_int(seed) + (tensor_id * GOLDEN & MASK64))


def h_tensor_id(step: int) -> int:
    return TID_H | (step << 8)


_CHUNK = 1 << 22


def raw_draws(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    key = stream_key(seed, tensor_id)
    out = np.empty(count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        for c0 in range(0, count, _CHUNK):
            c1 = min(count, c0 + _CHUNK)
            n = np.arange(start + c0 + 1, start + c1 + 1, dtype=np.uint64)
            out[c0:c1] = _mix_np(np.uint64(key) + n * np.uint64(GOLDEN))
    return out


def normal_scale(sigma: float) -> float:
    return float(sigma) * SQRT3_OVER_65536


def normal_f32(seed: int, tensor_id: int, start: int, count: int, sigma: float) -> np.ndarray:
    """float32 N(0, sigma^2) stand-ins (see module docstring)."""
    scale = normal_scale(sigma)
    out = np.empty(count, dtype=np.float32)
    for c0 in range(0, count, _CHUNK):
        c1 = min(count, c0 + _CHUNK)
        r = raw_draws(seed, tensor_id, start + c0, c1 - c0)
        s = (r & np.uint64(0xFFFF)) + ((r >> np.uint64(16)) & np.uint64(0xFFFF)) \
            + ((r >> np.uint64(32)) & np.uint64(0xFFFF)) + (r >> np.uint64(48))
        cen = s.astype(np.int64) - IRWIN_HALL_CENTRE
        out[c0:c1] = (cen.astype(np.float64) * scale).astype(np.float32)
    return out


def uniform_f32(seed: int, tensor_id: int, start: int, count: int, lo: float, hi: float) -> np.ndarray:
    r = raw_draws(seed, tensor_id, start, count)
    u = (r >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    width = float(hi) - float(lo)
    return (float(lo) + width * u).astype(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return b.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float32 values rounded to the nearest bf16 value, returned as float32."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    """Shape, routing rule and input recipe of one synthetic MoE-layer workload."""
    name: str
    T: int
    d_model: int
    E_r: int
    E_s: int
    K: int
    d_ffn: int
    d_ffn_shared: int
    score_fn: int          # 0 = sigmoid affinity, 1 = softmax
    dtype: str             # "f32", "bf16", or "bf16_e4m3" (bf16 activations, e4m3 expert weights)
    seed: int
    n_groups: int = 1
    topk_groups: int = 1
    group_topn: int = 0
    capacity_factor: float = 0.0
    add_residual: int = 1
    steps: int = 1
    gamma: float = 0.0
    bias_init: str = "zero"        # "zero" | "uniform_0.01"
    centroid_skew: str = "none"    # "none" | "mean_dir_0.5" | "zipf_1.2"
    centroid_sigma: float = 0.02

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def R(self) -> int:          # routed (token, slot) pairs = upper bound on kept rows
        return self.T * self.K


WORKLOADS = {
    # Toy aux-loss-free routing, fp32, 60 bias steps with gamma = 0.1.
    "toy_fp32": Workload("toy_fp32", T=512, d_model=64, E_r=8, E_s=0, K=2, d_ffn=128,
                         d_ffn_shared=0, score_fn=0, dtype="f32", seed=1000, steps=60,
                         gamma=0.1, centroid_skew="mean_dir_0.5"),
    # Mixtral-style coarse layer: softmax over 8 experts, top-2, no shared, no bias.
    "mixtral_8x14336": Workload("mixtral_8x14336", T=4096, d_model=4096, E_r=8, E_s=0, K=2,
                                d_ffn=14336, d_ffn_shared=0, score_fn=1, dtype="bf16", seed=1001),
    # Fine-grained + shared: 64 routed (f=1408) + 2 shared, top-8, fixed U(-0.01,0.01) bias.
    "finegrained_64x1408": Workload("finegrained_64x1408", T=8192, d_model=2048, E_r=64, E_s=2,
                                    K=8, d_ffn=1408, d_ffn_shared=1408, score_fn=0, dtype="bf16",
                                    seed=1002, bias_init="uniform_0.01"),
    # DeepSeek-V3 shape: 256 routed (f=2048) + 1 shared, top-8 in 4 of 8 groups, bias chain.
    "deepseek_v3": Workload("deepseek_v3", T=4096, d_model=7168, E_r=256, E_s=1, K=8,
                            d_ffn=2048, d_ffn_shared=2048, score_fn=0, dtype="bf16", seed=1003,
                            n_groups=8, topk_groups=4, group_topn=2, steps=20, gamma=0.001),
    # Decode-sized skewed DeepSeek-V3 layer: T=64, Zipf(1.2) centroid norms, b = 0.
    "deepseek_v3_decode": Workload("deepseek_v3_decode", T=64, d_model=7168, E_r=256, E_s=1, K=8,
                                   d_ffn=2048, d_ffn_shared=2048, score_fn=0, dtype="bf16",
                                   seed=1004, n_groups=8, topk_groups=4, group_topn=2,
                                   centroid_skew="zipf_1.2"),
}
# The fine-grained layer is also run with GShard capacity factor 1.25.
WORKLOADS["finegrained_64x1408_cf1.25"] = WORKLOADS["finegrained_64x1408"].with_(
    name="finegrained_64x1408_cf1.25", capacity_factor=1.25)
# The DeepSeek-V3 layers with e4m3 expert weights (the same bf16 weights,
# quantized per row): the weight-streaming regime with half the bytes.
WORKLOADS["deepseek_v3_e4m3"] = WORKLOADS["deepseek_v3"].with_(name="deepseek_v3_e4m3", dtype="bf16_e4m3")
WORKLOADS["deepseek_v3_decode_e4m3"] = WORKLOADS["deepseek_v3_decode"].with_(
    name="deepseek_v3_decode_e4m3", dtype="bf16_e4m3")


def _dtype_round(x: np.ndarray, dtype: str) -> np.ndarray:
    return round_bf16(x) if dtype != "f32" else x


def gen_h(w: Workload, step: int = 0, tokens: Optional[slice] = None) -> np.ndarray:
    """Token activations h [T, d] (float32 holding exact bf16 values for bf16 workloads)."""
    t0, t1 = (0, w.T) if tokens is None else (tokens.start, tokens.stop)
    x = normal_f32(w.seed, h_tensor_id(step), t0 * w.d_model, (t1 - t0) * w.d_model, 1.0)
    return _dtype_round(x, w.dtype).reshape(t1 - t0, w.d_model)


def gen_centroids(w: Workload) -> np.ndarray:
    """Router centroids e [E_r, d] float32, with the workload's skew applied."""
    e = normal_f32(w.seed, TID_E, 0, w.E_r * w.d_model, w.centroid_sigma).reshape(w.E_r, w.d_model)
    if w.centroid_skew == "mean_dir_0.5":
        # expert 0 gets +0.5 along the unit mean direction of the step-0 tokens
        mu = gen_h(w, 0).astype(np.float64).mean(axis=0)
        u = mu / np.linalg.norm(mu)
        e = e.copy()
        e[0] = (e[0].astype(np.float64) + 0.5 * u).astype(np.float32)
    elif w.centroid_skew == "zipf_1.2":
        rank_factor = np.arange(1, w.E_r + 1, dtype=np.float64) ** -1.2
        e = (e.astype(np.float64) * rank_factor[:, None]).astype(np.float32)
    return np.ascontiguousarray(e)


def gen_bias(w: Workload) -> np.ndarray:
    if w.bias_init == "uniform_0.01":
        return uniform_f32(w.seed, TID_B, 0, w.E_r, -0.01, 0.01)
    return np.zeros(w.E_r, dtype=np.float32)


def weight_spec(w: Workload, which: str):
    """(tensor_id, n_experts, rows, cols, sigma) of one stacked weight tensor.

    which: 'gate' | 'up' | 'down' (routed) or 'sgate' | 'sup' | 'sdown' (shared).
    Layouts follow nn.Linear: gate/up are [E, f, d], down is [E, d, f]; sigma is
    1/sqrt(fan_in).
    """
    d, f, fs = w.d_model, w.d_ffn, w.d_ffn_shared
    return {
        "gate": (TID_WG, w.E_r, f, d, 1.0 / math.sqrt(d)),
        "up": (TID_WU, w.E_r, f, d, 1.0 / math.sqrt(d)),
        "down": (TID_WD, w.E_r, d, f, 1.0 / math.sqrt(f) if f else 0.0),
        "sgate": (TID_WSG, w.E_s, fs, d, 1.0 / math.sqrt(d)),
        "sup": (TID_WSU, w.E_s, fs, d, 1.0 / math.sqrt(d)),
        "sdown": (TID_WSD, w.E_s, d, fs, 1.0 / math.sqrt(fs) if fs else 0.0),
    }[which]


def gen_weight(w: Workload, which: str, expert: Optional[int] = None) -> np.ndarray:
    """One stacked weight tensor [E, rows, cols], or one expert's slice [rows, cols]."""
    tid, n, rows, cols, sigma = weight_spec(w, which)
    per = rows * cols
    if expert is None:
        x = normal_f32(w.seed, tid, 0, n * per, sigma).reshape(n, rows, cols)
    else:
        x = normal_f32(w.seed, tid, expert * per, per, sigma).reshape(rows, cols)
    return _dtype_round(x, w.dtype)

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
* Normal variates: the Box-Muller transform (Box & Muller, "A note on the
  generation of random normal deviates", Ann. Math. Statist. 1958) of the two
  32-bit halves of one draw: u1 = (hi + 1/2) 2**-32 in (0, 1), u2 = lo 2**-32,
  z = sqrt(-2 ln u1) cos(2 pi u2), times sigma.  ln and cos are evaluated by
  fixed series in plain IEEE double operations, each rounded on its own (no
  library call, no fused multiply-add), so that the C and CUDA twins in
  ``gen.cu`` reproduce every value bit for bit:
  - ln x for x = hi + 1/2: x = m 2**e exactly with m in [sqrt(1/2), sqrt(2)),
    ln m = 2 atanh(s) = 2 s (1 + s^2/3 + s^4/5 + ... + s^20/21) with
    s = (m - 1)/(m + 1), |s| <= 0.172 (the truncated terms are below 2**-60
    relative), and ln u1 = ln m + (e - 32) ln 2;
  - cos(2 pi u2): the quadrant and the position in it come exactly from the
    integer lo; the angle is folded into [0, pi/4] (theta = g pi / 2**31 with
    g <= 2**29) and cos theta, sin theta are Taylor series to the theta^20 and
    theta^21 terms (the remainders are below 2**-70).
  The tails reach +-6.76 sigma (u1 >= 2**-33).
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

# Constants of the normal variates as exact double bit patterns (the same hex
# literals stand in gen.cu): ln 2, sqrt(1/2), pi / 2**31, and the series
# coefficients 1/(2k+1), (-1)^k/(2k)!, (-1)^k/(2k+1)! for k = 0..10.
_LN2 = float.fromhex("0x1.62e42fefa39efp-1")
_SQRT_HALF = float.fromhex("0x1.6a09e667f3bcdp-1")
_PI_OVER_2_31 = float.fromhex("0x1.921fb54442d18p-30")
_LN_C = [float.fromhex(h) for h in (
    "0x1.0000000000000p+0", "0x1.5555555555555p-2", "0x1.999999999999ap-3", "0x1.2492492492492p-3",
    "0x1.c71c71c71c71cp-4", "0x1.745d1745d1746p-4", "0x1.3b13b13b13b14p-4", "0x1.1111111111111p-4",
    "0x1.e1e1e1e1e1e1ep-5", "0x1.af286bca1af28p-5", "0x1.8618618618618p-5")]
_COS_C = [float.fromhex(h) for h in (
    "0x1.0000000000000p+0", "-0x1.0000000000000p-1", "0x1.5555555555555p-5", "-0x1.6c16c16c16c17p-10",
    "0x1.a01a01a01a01ap-16", "-0x1.27e4fb7789f5cp-22", "0x1.1eed8eff8d898p-29", "-0x1.93974a8c07c9dp-37",
    "0x1.ae7f3e733b81fp-45", "-0x1.6827863b97d97p-53", "0x1.e542ba4020225p-62")]
_SIN_C = [float.fromhex(h) for h in (
    "0x1.0000000000000p+0", "-0x1.5555555555555p-3", "0x1.1111111111111p-7", "-0x1.a01a01a01a01ap-13",
    "0x1.71de3a556c734p-19", "-0x1.ae64567f544e4p-26", "0x1.6124613a86d09p-33", "-0x1.ae7f3e733b81fp-41",
    "0x1.952c77030ad4ap-49", "-0x1.2f49b46814157p-57", "0x1.71b8ef6dcf572p-66")]

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


def _horner(coeffs, w: np.ndarray) -> np.ndarray:
    """c0 + w (c1 + w (c2 + ...)), one rounded multiply and one rounded add per step."""
    p = np.full_like(w, coeffs[-1])
    for c in reversed(coeffs[:-1]):
        p = p * w
        p = p + c
    return p


def ln_half_int(hi: np.ndarray) -> np.ndarray:
    """ln(hi + 1/2) - 32 ln 2 = ln(u1) for 32-bit integers hi (see module docstring)."""
    x = hi.astype(np.float64) + 0.5
    m, e = np.frexp(x)                         # x = m 2**e, m in [1/2, 1), exact
    low = m < _SQRT_HALF
    m = np.where(low, m * 2.0, m)
    e = np.where(low, e - 1, e)
    s = (m - 1.0) / (m + 1.0)
    p = _horner(_LN_C, s * s)
    return (s * 2.0) * p + (e - 32).astype(np.float64) * _LN2


def cos_2pi_frac(lo: np.ndarray) -> np.ndarray:
    """cos(2 pi lo / 2**32) for 32-bit integers lo (see module docstring)."""
    lo = lo.astype(np.int64)
    q = lo >> 30                               # quadrant
    f = lo & ((1 << 30) - 1)                   # position in it, angle f pi / 2**31
    fold = f >= (1 << 29)
    g = np.where(fold, (1 << 30) - f, f).astype(np.float64)
    th = g * _PI_OVER_2_31                     # in [0, pi/4]
    w = th * th
    c = _horner(_COS_C, w)
    sn = th * _horner(_SIN_C, w)
    ca = np.where(fold, sn, c)                 # cos and sin of the angle within the quadrant
    sa = np.where(fold, c, sn)
    return np.select([q == 0, q == 1, q == 2], [ca, -sa, -ca], sa)


def normal_f32(seed: int, tensor_id: int, start: int, count: int, sigma: float) -> np.ndarray:
    """float32 N(0, sigma^2) draws (Box-Muller; see module docstring)."""
    out = np.empty(count, dtype=np.float32)
    sig = float(sigma)
    for c0 in range(0, count, _CHUNK):
        c1 = min(count, c0 + _CHUNK)
        r = raw_draws(seed, tensor_id, start + c0, c1 - c0)
        rad = np.sqrt(ln_half_int(r >> np.uint64(32)) * -2.0)
        z = rad * cos_2pi_frac(r & np.uint64(0xFFFFFFFF))
        out[c0:c1] = (z * sig).astype(np.float32)
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

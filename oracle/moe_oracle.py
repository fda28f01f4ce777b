"""CPU oracle for the forward pass of one sparse MoE layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library; its inputs come from ``moe_inputs``.

It is a plain, slow restatement of what the source pages define, in float64
wherever the pages do not fix the precision, and in float32 exactly where the
method itself works in fp32 (the biased selection key s + b, the gate
normalisation and the bias step).  Library primitives used as single steps:
numpy matmul, stable argsort, bincount.

Sources (web pages, cited by title and section/equation):

[SMoE]  "Sparse Mixture-of-Experts (MoE): Routing Math, Load Balancing & Expert
        Parallelism" -- section 0 equation "Fine-Grained + Shared Expert MoE Layer
        Output"; section 1 (ClassicalTopKRouter: softmax, top-K, renormalise);
        section 2 equation "Auxiliary-Loss-Free Biased Selection & Unbiased Gate
        Aggregation" (selection on s + b, gates from s, counts, c-bar, sign step);
        section 3 "Expert Buffer Capacity & Token Dropping Bound";
        section 4 item 1 (MaxVio).
[RLB]   "Mixture of Experts: Routing and Load Balancing" -- section 2 "The
        routing rule, exactly"; section 5 "One property that is deliberately
        false" (capacity admits tokens in the order they appear).
[EPLB]  "Mixture-of-Experts: Expert Parallelism, All-to-All Routing, and
        Auxiliary-Loss-Free Load Balancing" -- "Expert Parallelism and All-to-All
        Communication" (capacity buffers, overflow dropped).
[DS3LB] "Load Balancing -- DeepSeek-V3" -- "How it works" (g' and g equations,
        fair share K_r T / N_r); "Official code" (bias added before grouped top-k).
[GMF]   "GPUs, memory and failures" -- the worked bias example (MaxVio 2.0,
        gamma = 0.1) and the bias card (route_with_bias / update_bias /
        log_router).

Readings where the pages are silent or disagree (each is also listed in the
design notes):
  * top-K ties go to the lower expert index; group ties to the lower group index;
  * the selected set I_t is stored in ascending expert index, and the gate
    denominator is summed in that order in fp32;
  * sign(0) = 0, evaluated exactly in integers as sign(K*T - E_r*c_i);
  * capacity C = floor(T*K*CF/E_r) with CF taken as an fp32 value; overflow keeps
    the lowest token indices; counts for the bias are pre-drop;
  * group-limited selection: a group's score is the fp32 sum of its top
    ``group_topn`` keys taken in descending order; experts outside the kept
    groups are ineligible (-inf), never 0;
  * the sigmoid affinity is evaluated from fp32 logits in double and rounded to
    fp32; softmax likewise.

Pins (see tests/test_oracle_pins.py): the worked bias example, brute-force
subset enumeration, the softmax closed form, gate/count/bias invariants,
reductions to a dense SwiGLU FFN computed with torch.nn.functional, a dense
all-experts restatement of the layer equation, and planted-mistake tests.
The expert FFN values themselves have no printed values on the pages: beyond
those reductions they are "parity unpinned".

Router losses and logging (aux_loss, z_loss, seq_balance_loss, load_entropy,
dropped_rate) are pinned in tests/test_oracle_router_stats.py.  The e4m3
quantization of expert weights and rows (e4m3_encode, pow2_scale,
quantize_rows, swiglu_q8, layer_output_q8) is pinned in
tests/test_oracle_fp8.py against torch's float8_e4m3fn conversion, ties to
even, the closed form of the scale and the format's error bound; the
quantized expert's values beyond that bound are "parity unpinned".
The layer backward (swiglu_backward, gate_backward, score_backward,
layer_backward) is pinned in tests/test_oracle_backward.py against
torch.autograd through a dense restatement of the forward, finite
differences, and planted mistakes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Callable, Dict, Optional

import numpy as np

F32 = np.float32
GATE_EPS = F32(1e-12)


# ---------------------------------------------------------------------------
# a1: router affinity  ([SMoE] section 2, s = sigmoid(h . e); section 1 softmax)
# ---------------------------------------------------------------------------

def router_logits(h: np.ndarray, e: np.ndarray) -> np.ndarray:
    """z[t, i] = h_t . e_i, accumulated in float64 and rounded once to fp32."""
    return (np.asarray(h, np.float64) @ np.asarray(e, np.float64).T).astype(F32)


def sigmoid_scores(z32: np.ndarray) -> np.ndarray:
    """s = sigma(z) evaluated in double from the fp32 logit, rounded to fp32."""
    z = z32.astype(np.float64)
    with np.errstate(over="ignore"):
        return (1.0 / (1.0 + np.exp(-z))).astype(F32)


def softmax_scores(z32: np.ndarray) -> np.ndarray:
    """p = softmax(z) over the experts, in double, rounded to fp32."""
    z = z32.astype(np.float64)
    ez = np.exp(z - z.max(axis=1, keepdims=True))
    return (ez / ez.sum(axis=1, keepdims=True)).astype(F32)


def affinity(h: np.ndarray, e: np.ndarray, score_fn: int) -> np.ndarray:
    z = router_logits(h, e)
    return sigmoid_scores(z) if score_fn == 0 else softmax_scores(z)


# ---------------------------------------------------------------------------
# a2: selection I_t = TopK(s + b) with optional group limit ([SMoE] s.2, [DS3LB])
# ---------------------------------------------------------------------------

def selection_keys(s32: np.ndarray, b32: np.ndarray) -> np.ndarray:
    """key = s + b as one fp32 add (the bias only picks, it never scales)."""
    return (s32.astype(F32) + np.asarray(b32, F32)[None, :]).astype(F32)


def group_scores(keys: np.ndarray, n_groups: int, group_topn: int) -> np.ndarray:
    """Score of each group of E_r/n_groups consecutive experts: the fp32 sum of
    its group_topn largest keys, added in descending order."""
    T, E = keys.shape
    kg = keys.reshape(T, n_groups, E // n_groups)
    desc = -np.sort(-kg, axis=2)          # descending within each group
    G = desc[:, :, 0].astype(F32)
    for j in range(1, group_topn):
        G = (G + desc[:, :, j]).astype(F32)
    return G


def eligible_mask(keys: np.ndarray, n_groups: int, topk_groups: int, group_topn: int) -> np.ndarray:
    """Experts in the topk_groups best groups (ties -> lower group index)."""
    T, E = keys.shape
    if n_groups <= 1 or group_topn <= 0:
        return np.ones((T, E), dtype=bool)
    G = group_scores(keys, n_groups, group_topn)
    order = np.argsort(-G, axis=1, kind="stable")[:, :topk_groups]
    keep_g = np.zeros((T, n_groups), dtype=bool)
    np.put_along_axis(keep_g, order, True, axis=1)
    return np.repeat(keep_g, E // n_groups, axis=1)


def select_experts(s32: np.ndarray, b32: np.ndarray, K: int, n_groups: int = 1,
                   topk_groups: int = 1, group_topn: int = 0) -> np.ndarray:
    """I_t: the K eligible experts with the largest key (ties -> lower index),
    returned in ascending expert index, int32 [T, K]."""
    keys = selection_keys(s32, b32)
    elig = eligible_mask(keys, n_groups, topk_groups, group_topn)
    masked = np.where(elig, keys, F32(-np.inf)).astype(F32)
    order = np.argsort(-masked, axis=1, kind="stable")[:, :K]
    return np.sort(order, axis=1).astype(np.int32)


# ---------------------------------------------------------------------------
# a3: gates g = s_i / sum_{j in I_t} s_j  ([SMoE] s.2; [DS3LB] g = g'/sum g')
# ---------------------------------------------------------------------------

def gates_from_scores(s32: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Unbiased gates in fp32; the denominator is summed in ascending expert
    index and clamped at 1e-12 (the clamp of the pages' router code)."""
    sel = np.take_along_axis(s32.astype(F32), idx.astype(np.int64), axis=1)
    S = sel[:, 0].astype(F32)
    for k in range(1, idx.shape[1]):
        S = (S + sel[:, k]).astype(F32)
    return (sel / np.maximum(S, GATE_EPS)[:, None]).astype(F32)


# ---------------------------------------------------------------------------
# a4 / a9: load counts, MaxVio, bias step  ([SMoE] s.2 and s.4; [GMF])
# ---------------------------------------------------------------------------

def load_counts(idx: np.ndarray, E_r: int) -> np.ndarray:
    """c_i = number of tokens whose selected set contains i (before any drop)."""
    return np.bincount(idx.reshape(-1).astype(np.int64), minlength=E_r).astype(np.int64)


def max_vio(counts: np.ndarray, K: int, T: int, E_r: int) -> float:
    """MaxVio = (max_i c_i - c_bar) / c_bar with c_bar = K*T/E_r."""
    cbar = K * T / E_r
    return float((counts.max() - cbar) / cbar)


def bias_update(b32: np.ndarray, counts: np.ndarray, K: int, T: int, gamma: float) -> np.ndarray:
    """b_i <- b_i + gamma * sign(c_bar - c_i): the sign is taken exactly in
    integers as sign(K*T - E_r*c_i) (sign(0) = 0), the step is one fp32 add."""
    E_r = counts.shape[0]
    sgn = np.sign(K * T - E_r * counts.astype(np.int64)).astype(F32)
    return (np.asarray(b32, F32) + F32(gamma) * sgn).astype(F32)


# ---------------------------------------------------------------------------
# a5: dispatch / permutation with optional capacity ([SMoE] s.3; [EPLB]; [RLB] s.5)
# ---------------------------------------------------------------------------

def capacity(T: int, K: int, E_r: int, capacity_factor: float) -> int:
    """floor(T*K*CF/E_r) for CF > 0 (CF read as an fp32 value); T*K when dropless."""
    cf = float(np.float32(capacity_factor))
    if cf <= 0.0:
        return T * K
    return int(math.floor(float(T * K) * cf / float(E_r)))


@dataclass
class Dispatch:
    counts: np.ndarray     # [E_r] pre-drop selection counts
    kept: np.ndarray       # [E_r] rows kept per expert
    offsets: np.ndarray    # [E_r + 1] exclusive scan of kept
    perm_tok: np.ndarray   # [sum kept] token of each permuted row
    perm_slot: np.ndarray  # [sum kept] slot k of each permuted row
    row_of: np.ndarray     # [T, K] permuted row of (t, k), -1 when dropped


def dispatch(idx: np.ndarray, E_r: int, capacity_factor: float = 0.0) -> Dispatch:
    """Rows grouped by expert (ascending), tokens ascending within an expert; at
    most C rows per expert, the lowest token indices admitted first."""
    T, K = idx.shape
    C = capacity(T, K, E_r, capacity_factor)
    t_of = np.repeat(np.arange(T, dtype=np.int64), K)
    k_of = np.tile(np.arange(K, dtype=np.int64), T)
    e_of = idx.reshape(-1).astype(np.int64)
    order = np.argsort(e_of * T + t_of, kind="stable")
    counts = load_counts(idx, E_r)
    kept = np.minimum(counts, C)
    offsets = np.zeros(E_r + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    starts = np.zeros(E_r + 1, dtype=np.int64)
    starts[1:] = np.cumsum(counts)
    row_of = np.full((T, K), -1, dtype=np.int64)
    perm_tok = np.empty(int(offsets[-1]), dtype=np.int64)
    perm_slot = np.empty(int(offsets[-1]), dtype=np.int64)
    for ex in range(E_r):
        seg = order[starts[ex]:starts[ex] + kept[ex]]
        rows = offsets[ex] + np.arange(kept[ex])
        perm_tok[rows] = t_of[seg]
        perm_slot[rows] = k_of[seg]
        row_of[t_of[seg], k_of[seg]] = rows
    return Dispatch(counts, kept, offsets, perm_tok, perm_slot, row_of)


# ---------------------------------------------------------------------------
# a6 / a7: SwiGLU expert ([SMoE] s.0: SwiGLU(h) = (SiLU(h W_gate) * (h W_up)) W_down)
# ---------------------------------------------------------------------------

def swiglu(x: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """One SwiGLU expert in float64.  Weights use the nn.Linear layout:
    w_gate, w_up [f, d]; w_down [d, f]."""
    x = np.asarray(x, np.float64)
    u = x @ np.asarray(w_gate, np.float64).T
    v = x @ np.asarray(w_up, np.float64).T
    with np.errstate(over="ignore"):
        a = u / (1.0 + np.exp(-u)) * v          # SiLU(u) * v
    return a @ np.asarray(w_down, np.float64).T


# ---------------------------------------------------------------------------
# a8: the layer equation ([SMoE] s.0)
#   y_t = h_t + sum_j SwiGLU^S_j(h_t) + sum_{i in TopK} g_{t,i} SwiGLU^R_i(h_t)
# ---------------------------------------------------------------------------

WeightSource = Callable[[str, int], np.ndarray]   # (which, expert) -> 2-D weight


@dataclass
class LayerConfig:
    T: int
    d_model: int
    E_r: int
    E_s: int
    K: int
    score_fn: int = 0
    n_groups: int = 1
    topk_groups: int = 1
    group_topn: int = 0
    capacity_factor: float = 0.0
    add_residual: int = 1


def route(cfg: LayerConfig, s32: np.ndarray, b32: np.ndarray):
    """Selection, gates and dispatch from given fp32 scores (a2-a5)."""
    idx = select_experts(s32, b32, cfg.K, cfg.n_groups, cfg.topk_groups, cfg.group_topn)
    gates = gates_from_scores(s32, idx)
    disp = dispatch(idx, cfg.E_r, cfg.capacity_factor)
    return idx, gates, disp


def layer_output(cfg: LayerConfig, h: np.ndarray, idx: np.ndarray, gates: np.ndarray,
                 disp: Dispatch, weights: WeightSource,
                 tokens: Optional[np.ndarray] = None) -> np.ndarray:
    """y for the given tokens (all tokens when None), float64 [n, d].

    Expert i is evaluated on exactly the kept (t, i) pairs among those tokens;
    dropped pairs contribute nothing and the surviving gates are not
    renormalised."""
    tok = np.arange(cfg.T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    x = np.asarray(h, np.float64)[tok]
    y = x * float(cfg.add_residual)
    for j in range(cfg.E_s):
        y = y + swiglu(x, weights("sgate", j), weights("sup", j), weights("sdown", j))
    kept = disp.row_of[tok] >= 0                       # [n, K]
    ex_of = idx[tok].astype(np.int64)
    for ex in np.unique(ex_of[kept]):
        rows, ks = np.nonzero((ex_of == ex) & kept)
        o = swiglu(x[rows], weights("gate", ex), weights("up", ex), weights("down", ex))
        y[rows] += gates[tok[rows], ks].astype(np.float64)[:, None] * o
    return y


def layer_forward(cfg: LayerConfig, h: np.ndarray, e: np.ndarray, b32: np.ndarray,
                  weights: WeightSource, s_in: Optional[np.ndarray] = None,
                  tokens: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Whole layer: affinity (or the given fp32 scores s_in), selection, gates,
    dispatch and the output y (for ``tokens`` only, when given)."""
    s32 = affinity(h, e, cfg.score_fn) if s_in is None else np.asarray(s_in, F32)
    b_sel = np.asarray(b32, F32) if cfg.score_fn == 0 else np.zeros(cfg.E_r, F32)
    idx, gates, disp = route(cfg, s32, b_sel)
    y = layer_output(cfg, h, idx, gates, disp, weights, tokens)
    return dict(s=s32, idx=idx, gates=gates, counts=disp.counts, kept=disp.kept,
                offsets=disp.offsets, perm_tok=disp.perm_tok, row_of=disp.row_of, y=y,
                max_vio=max_vio(disp.counts, cfg.K, cfg.T, cfg.E_r))


def array_weights(wg, wu, wd, swg=None, swu=None, swd=None) -> WeightSource:
    """WeightSource over stacked arrays [E, rows, cols]."""
    table = dict(gate=wg, up=wu, down=wd, sgate=swg, sup=swu, sdown=swd)
    return lambda which, ex: table[which][ex]


# ---------------------------------------------------------------------------
# Independent-routing agreement: the tokens whose selection is numerically
# fragile (K-th vs (K+1)-th eligible key gap, and the last kept vs first
# dropped group score gap, below a threshold).
# ---------------------------------------------------------------------------

def near_tie_tokens(s32: np.ndarray, b32: np.ndarray, K: int, n_groups: int = 1,
                    topk_groups: int = 1, group_topn: int = 0, gap: float = 1e-5) -> np.ndarray:
    keys = selection_keys(s32, b32).astype(np.float64)
    T, E = keys.shape
    fragile = np.zeros(T, dtype=bool)
    if n_groups > 1 and group_topn > 0 and topk_groups < n_groups:
        G = np.sort(group_scores(selection_keys(s32, b32), n_groups, group_topn).astype(np.float64), axis=1)[:, ::-1]
        fragile |= (G[:, topk_groups - 1] - G[:, topk_groups]) < gap
    elig = eligible_mask(selection_keys(s32, b32), n_groups, topk_groups, group_topn)
    masked = np.where(elig, keys, -np.inf)
    srt = -np.sort(-masked, axis=1)
    if K < E:
        nxt = srt[:, K]
        fragile |= np.isfinite(nxt) & ((srt[:, K - 1] - nxt) < gap)
    return fragile


# ---------------------------------------------------------------------------
# Router losses and logging ([SMoE] section 1 "Switch Auxiliary Loss & ST-MoE
# Router z-Loss" equations; [DS3LB] "How it works", sequence-wise L_Bal;
# [GMF] the bias card's log_router: MaxVio, dropped rate, router entropy)
# ---------------------------------------------------------------------------

def normalized_scores(s32: np.ndarray) -> np.ndarray:
    """s'_{t,i} = s_{t,i} / sum_j s_{t,j} over all experts (equals p for softmax)."""
    s = np.asarray(s32, np.float64)
    return s / s.sum(axis=1, keepdims=True)


def aux_loss(s32: np.ndarray, idx: np.ndarray, E_r: int, K: int, alpha: float) -> float:
    """Switch auxiliary loss alpha * sum_i f_i P_i, f_i = E_r/(K T) * c_i,
    P_i = mean_t s'_{t,i}."""
    T = idx.shape[0]
    f = E_r / (K * T) * load_counts(idx, E_r).astype(np.float64)
    P = normalized_scores(s32).mean(axis=0)
    return float(alpha * np.sum(f * P))


def z_loss(z32: np.ndarray, c_z: float) -> float:
    """Router z-loss c_z / T * sum_t (log sum_i exp z_{t,i})^2."""
    z = np.asarray(z32, np.float64)
    m = z.max(axis=1, keepdims=True)
    lse = (m + np.log(np.exp(z - m).sum(axis=1, keepdims=True)))[:, 0]
    return float(c_z * np.mean(lse ** 2))


def seq_balance_loss(s32: np.ndarray, idx: np.ndarray, E_r: int, K: int, seq_len: int,
                     alpha: float) -> float:
    """Sequence-wise balance loss, averaged over the T/seq_len sequences:
    alpha * sum_i f_i P_i per sequence, with f_i = E_r/(K S) * (selections of i
    in the sequence) and P_i = mean over the sequence of s'_{t,i}."""
    T = idx.shape[0]
    sp = normalized_scores(s32)
    total = 0.0
    n_seq = T // seq_len
    for b in range(n_seq):
        rows = slice(b * seq_len, (b + 1) * seq_len)
        f = E_r / (K * seq_len) * load_counts(idx[rows], E_r).astype(np.float64)
        P = sp[rows].mean(axis=0)
        total += alpha * np.sum(f * P)
    return float(total / n_seq)


def load_entropy(counts: np.ndarray) -> float:
    """Entropy of the load shares, -sum share * log(max(share, 1e-9))."""
    share = np.asarray(counts, np.float64) / np.sum(counts)
    return float(-np.sum(share * np.log(np.maximum(share, 1e-9))))


def dropped_rate(kept: np.ndarray, counts: np.ndarray) -> float:
    """Fraction of (token, expert) pairs dropped by capacity, 1 - kept/selected."""
    return float(1.0 - np.sum(kept) / np.sum(counts))


# ---------------------------------------------------------------------------
# Low-precision expert weights ([GMF] suggests keeping expert weights at lower
# precision when serving is bound by streaming them).  The pages name no format; the reading here (also
# in the design notes): fp8 e4m3 codes (1 sign, 4 exponent bits with bias 7,
# 3 mantissa bits, no infinities, largest finite 448) with one power-of-two
# scale per weight row (output channel) and per activation row (token); the
# tensor cores multiply e4m3 by e4m3, so the rows entering each GEMM are
# quantized the same way.  A scale is the smallest power of two s with
# amax / s <= 448, so x / s is exact and the only rounding is e4m3's own
# (to nearest, ties to the even code, saturating at +-448).
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_table() -> np.ndarray:
    """Values of the non-negative finite e4m3 codes 0..126 (ascending)."""
    codes = np.arange(127)
    e, m = codes >> 3, codes & 7
    return np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))


def e4m3_encode(x32: np.ndarray) -> np.ndarray:
    """uint8 e4m3 codes of fp32 values: nearest finite value, ties to the even
    code, |x| >= 448 saturates to 448; the sign bit is x's (a negative value
    that rounds to zero gives -0, code 0x80)."""
    x = np.asarray(x32, np.float64)
    tab = e4m3_table()
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(tab, a, side="left"), 0, 126)    # first value >= a
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - tab[lo], tab[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    sign = np.signbit(x).astype(np.uint8) << 7                      # -0 keeps its sign, as in IEEE
    return (code | sign).astype(np.uint8)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, np.uint8)
    v = e4m3_table()[np.minimum(c & 0x7F, 126)]
    return np.where(c & 0x80, -v, v)


def pow2_scale(amax32: np.ndarray) -> np.ndarray:
    """Smallest power of two s with amax / s <= 448, as fp32 (1 where amax == 0),
    and never below 2^-126 (a scale is a normal fp32 number).
    With amax = M * 2^E (1 <= M < 2): s = 2^max(E - 8 + [M > 1.75], -126)."""
    a = np.asarray(amax32, np.float64)
    m, ex = np.frexp(a)                     # a = m * 2^ex, 0.5 <= m < 1
    e = np.maximum((ex - 1) - 8 + (2.0 * m > 1.75), -126)
    return np.where(a > 0, np.ldexp(1.0, e), 1.0).astype(F32)


def quantize_rows(x32: np.ndarray):
    """Per-row power-of-two scale and e4m3 codes of an fp32 matrix [n, c]."""
    x = np.asarray(x32, F32)
    s = pow2_scale(np.max(np.abs(x), axis=1) if x.shape[1] else np.zeros(x.shape[0], F32))
    codes = e4m3_encode(x.astype(np.float64) / s.astype(np.float64)[:, None])
    return codes, s


def dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    return e4m3_decode(codes) * np.asarray(scales, np.float64)[:, None]


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (to nearest even) through torch's conversion; float64 out."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(x, np.float64)))
    return t.to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def swiglu_q8(x: np.ndarray, wg, wu, wd) -> np.ndarray:
    """One SwiGLU expert with e4m3 weights: wg, wu, wd are (codes, scales) with
    the nn.Linear layout.  The input rows are quantized per row, the products
    accumulate in float64, the SwiGLU product A is stored in bf16 and quantized
    per row before the down projection."""
    xq = dequantize_rows(*quantize_rows(np.asarray(x, F32)))
    u = xq @ dequantize_rows(*wg).T
    v = xq @ dequantize_rows(*wu).T
    with np.errstate(over="ignore"):
        a = bf16_round(u / (1.0 + np.exp(-u)) * v)
    aq = dequantize_rows(*quantize_rows(a.astype(F32)))
    return aq @ dequantize_rows(*wd).T


def layer_output_q8(cfg: LayerConfig, h: np.ndarray, idx: np.ndarray, gates: np.ndarray,
                    disp: Dispatch, weights, tokens: Optional[np.ndarray] = None) -> np.ndarray:
    """layer_output with e4m3 expert weights; ``weights(which, ex)`` returns
    (codes, scales).  Same layer equation, experts evaluated by swiglu_q8."""
    tok = np.arange(cfg.T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    x = np.asarray(h, np.float64)[tok]
    y = x * float(cfg.add_residual)
    for j in range(cfg.E_s):
        y = y + swiglu_q8(x, weights("sgate", j), weights("sup", j), weights("sdown", j))
    kept = disp.row_of[tok] >= 0
    ex_of = idx[tok].astype(np.int64)
    for ex in np.unique(ex_of[kept]):
        rows, ks = np.nonzero((ex_of == ex) & kept)
        o = swiglu_q8(x[rows], weights("gate", ex), weights("up", ex), weights("down", ex))
        y[rows] += gates[tok[rows], ks].astype(np.float64)[:, None] * o
    return y


# ---------------------------------------------------------------------------
# Backward pass of the layer ([SMoE] section 2: the selection uses s + b but
# the gates g are built from s alone, so the gradient reaches the router
# through g and never reaches the bias; [EPLB]: the bias is a buffer updated
# by the sign rule, not by gradient descent).  The selected set I_t and the
# capacity decisions are piecewise constant: no gradient flows through them.
# Everything in float64.
# ---------------------------------------------------------------------------

def swiglu_backward(x, w_gate, w_up, w_down, d_out):
    """Gradients of one SwiGLU expert o = (SiLU(x Wg^T) * (x Wu^T)) Wd^T for
    rows x [n, d] and the output gradient d_out [n, d]:
    (dx, dWg, dWu, dWd, o) -- o is returned for the gate gradient."""
    x = np.asarray(x, np.float64)
    wg, wu, wd = (np.asarray(w, np.float64) for w in (w_gate, w_up, w_down))
    do = np.asarray(d_out, np.float64)
    u = x @ wg.T
    v = x @ wu.T
    sig = 1.0 / (1.0 + np.exp(-u))
    a = u * sig * v
    da = do @ wd                                   # dL/da  [n, f]
    du = da * v * sig * (1.0 + u * (1.0 - sig))    # SiLU'(u) = sig (1 + u (1 - sig))
    dv = da * u * sig
    dx = du @ wg + dv @ wu
    return dx, du.T @ x, dv.T @ x, do.T @ a, a @ wd.T


def gate_backward(s32: np.ndarray, idx: np.ndarray, dg: np.ndarray) -> np.ndarray:
    """dL/ds [T, E] from dL/dg [T, K] with g_k = s_{I_k} / max(S, 1e-12),
    S = sum_k s_{I_k}: ds_j = (dg_j - sum_k g_k dg_k) / S for j in I_t (the
    clamp inactive), ds_j = dg_j / 1e-12 when it is active, 0 outside I_t."""
    s = np.asarray(s32, np.float64)
    T = s.shape[0]
    sel = np.take_along_axis(s, idx.astype(np.int64), axis=1)
    S = sel.sum(axis=1)
    den = np.maximum(S, float(GATE_EPS))
    g = sel / den[:, None]
    dg = np.asarray(dg, np.float64)
    corr = np.where(S > float(GATE_EPS), (g * dg).sum(axis=1), 0.0)
    ds = np.zeros_like(s)
    np.put_along_axis(ds, idx.astype(np.int64), (dg - corr[:, None]) / den[:, None], axis=1)
    return ds


def score_backward(s32: np.ndarray, ds: np.ndarray, score_fn: int) -> np.ndarray:
    """dL/dz from dL/ds: sigmoid s(1 - s); softmax p * (ds - <ds, p>)."""
    s = np.asarray(s32, np.float64)
    if score_fn == 0:
        return ds * s * (1.0 - s)
    return s * (ds - (ds * s).sum(axis=1, keepdims=True))


def layer_backward(cfg: LayerConfig, h: np.ndarray, e: np.ndarray, s32: np.ndarray,
                   idx: np.ndarray, gates: np.ndarray, disp: Dispatch, weights: WeightSource,
                   dy: np.ndarray):
    """Gradients of the layer output y w.r.t. h, the centroids e and every
    expert weight, for the routing (idx, gates, disp) of the forward pass and
    dL/dy.  Returns dict(dh, de, dg, grads) with grads[(which, expert)]."""
    x = np.asarray(h, np.float64)
    dy = np.asarray(dy, np.float64)
    dh = dy * float(cfg.add_residual)
    grads = {}
    for j in range(cfg.E_s):
        dx, dwg, dwu, dwd, _ = swiglu_backward(x, weights("sgate", j), weights("sup", j),
                                               weights("sdown", j), dy)
        dh = dh + dx
        grads[("sgate", j)], grads[("sup", j)], grads[("sdown", j)] = dwg, dwu, dwd
    dg = np.zeros((cfg.T, cfg.K))
    kept = disp.row_of >= 0
    ex_of = idx.astype(np.int64)
    for ex in np.unique(ex_of[kept]):
        rows, ks = np.nonzero((ex_of == ex) & kept)
        g = gates[rows, ks].astype(np.float64)[:, None]
        dx, dwg, dwu, dwd, o = swiglu_backward(x[rows], weights("gate", ex), weights("up", ex),
                                               weights("down", ex), g * dy[rows])
        np.add.at(dh, rows, dx)
        dg[rows, ks] = (dy[rows] * o).sum(axis=1)
        grads[("gate", ex)], grads[("up", ex)], grads[("down", ex)] = dwg, dwu, dwd
    dz = score_backward(s32, gate_backward(s32, idx, dg), cfg.score_fn)
    dh = dh + dz @ np.asarray(e, np.float64)
    de = dz.T @ x
    return dict(dh=dh, de=de, dg=dg, dz=dz, grads=grads)

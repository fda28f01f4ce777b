#!/usr/bin/env python
"""Benchmark of the MoE layer forward on B200: tokens/s of the whole hot path
(routing, dispatch, grouped SwiGLU experts, combine, bias step) at the
DeepSeek-V3 shape, with the roofline fraction of its dominant kernel.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = moe_layer_forward over one fresh batch of T tokens followed by the
aux-loss-free bias step (the bias is carried from step to step).  Inputs are
synthetic (moe_inputs) and resident in HBM before the timed region; the expert
weights (22.6 GB) are far larger than L2, so no flush is needed.  N > 1 runs N
independent replicas (one process per GPU, no collective in the data path):
weak scaling, timed as the max over ranks.

At N = 1 the line also carries "workloads": one sub-record per other
configuration (decode-sized DeepSeek-V3, Mixtral-style, fine-grained dropless
and with capacity factor 1.25, the fp32 toy), each timed alone on the same GPU
with its own layer roofline, kernel rooflines and clocks (--workloads none
skips them).

Roofline bytes follow the definition: touched expert weights, shared weights,
centroids, h in and y out for the layer; for the gate/up GEMM (the dominant
kernel) its touched weights and h read once.  Permuted copies and
intermediates are implementation costs and are reported separately.

--impl reference times the CPU oracle (oracle/) on the host cores on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

METRIC = "MoE-layer fwd tokens/s @DeepSeek-V3 shape; % of bf16 tensor/HBM roofline"
DEFAULT_WORKLOAD = "deepseek_v3"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------------------
# algorithmic work of the layer and of its kernels
# ---------------------------------------------------------------------------

def layer_work(w, kept: np.ndarray):
    """(flops, bytes) of one layer step by the roofline definition: router
    GEMM + SwiGLU of every kept row and shared row; touched expert weights,
    shared weights, centroids, h in and y out."""
    n_rows = int(kept.sum())
    touched = int((kept > 0).sum())
    d, f, fs = w.d_model, w.d_ffn, w.d_ffn_shared
    flops = 2 * d * w.E_r * w.T + 6 * d * f * n_rows + 6 * d * fs * w.E_s * w.T
    es = 2 if w.dtype != "f32" else 4
    if w.dtype == "bf16_e4m3":
        # one byte per weight plus one fp32 scale per weight row
        wbytes = touched * (3 * d * f + 4 * (2 * f + d)) + w.E_s * (3 * d * fs + 4 * (2 * fs + d))
    else:
        wbytes = touched * 3 * d * f * es + w.E_s * 3 * d * fs * es
    nbytes = wbytes + w.E_r * d * 4 + 2 * w.T * d * es
    return flops, nbytes


def _weight_bytes(w, rows: int, cols: int) -> int:
    """Bytes of one expert weight matrix [rows, cols]: bf16 (2 B), fp32 (4 B), or
    e4m3 codes (1 B) plus one fp32 scale per row."""
    if w.dtype == "bf16_e4m3":
        return rows * cols + 4 * rows
    return rows * cols * (4 if w.dtype == "f32" else 2)


def gateup_work(w, kept: np.ndarray):
    """(flops, bytes) of one launch of the gate/up grouped GEMM by the roofline
    definition: the gate and up weights of every touched routed expert and of
    the shared experts, and the token rows h read once.  The permuted copy of
    the rows and the SwiGLU products are implementation costs, not counted."""
    n_rows = int(kept.sum())
    touched = int((kept > 0).sum())
    d, f, fs = w.d_model, w.d_ffn, w.d_ffn_shared
    flops = 4 * d * (f * n_rows + fs * w.E_s * w.T)
    es = 4 if w.dtype == "f32" else 2
    nbytes = 2 * touched * _weight_bytes(w, f, d) + 2 * w.E_s * _weight_bytes(w, fs, d) + w.T * d * es
    return flops, nbytes


def down_work(w, kept: np.ndarray):
    """(flops, bytes) of one launch of the down grouped GEMM by the roofline
    definition: the W_down of every touched routed expert and of the shared
    experts, and the layer output written once."""
    n_rows = int(kept.sum())
    touched = int((kept > 0).sum())
    d, f, fs = w.d_model, w.d_ffn, w.d_ffn_shared
    flops = 2 * d * (f * n_rows + fs * w.E_s * w.T)
    es = 4 if w.dtype == "f32" else 2
    nbytes = touched * _weight_bytes(w, d, f) + w.E_s * _weight_bytes(w, d, fs) + w.T * d * es
    return flops, nbytes


def gateup_impl_bytes(w, kept: np.ndarray) -> int:
    """Bytes the gate/up launch moves as implemented: the weights, one read of
    every permuted row (and of h for the shared experts) and one write of the
    SwiGLU products (the basis of the DRAM-traffic ratio in profiles/)."""
    n_rows = int(kept.sum())
    touched = int((kept > 0).sum())
    d, f, fs = w.d_model, w.d_ffn, w.d_ffn_shared
    rows_s = w.E_s * w.T
    if w.dtype == "bf16_e4m3":
        x_rows = n_rows + min(rows_s, w.T)
        return (touched * 2 * (d * f + 4 * f) + w.E_s * 2 * (d * fs + 4 * fs) + x_rows * (d + 4)
                + 2 * (n_rows * f + rows_s * fs))
    return 2 * (touched * 2 * d * f + w.E_s * 2 * d * fs + (n_rows + min(rows_s, w.T)) * d
                + n_rows * f + rows_s * fs)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi samples every 20 ms from construction on (nvidia-smi needs
    ~0.1 s to start, longer than a timed region); summary() keeps only the
    samples whose timestamps fall inside the window passed to mark()."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.window = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, window=None):
        import datetime
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != 8:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), float(parts[2]), parts[4:]))
            except ValueError:
                continue
        window = window or self.window
        if window:
            lo, hi = window
            inside = [r for r in rows if lo <= r[0] <= hi]
        else:
            inside = rows
        if not inside:
            return {"samples": 0, "note": "no nvidia-smi sample fell inside the timed region"}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, _, r in inside for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 0) for p in threadpool_info() if p.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


_WCACHE = __import__("collections").OrderedDict()   # (which, expert) -> host weights
_WCACHE_MAX = 192


def oracle_sample_time(w, tokens: np.ndarray, step: int = 0):
    """Time the oracle's layer forward (affinity, selection, gates, dispatch,
    experts, combine) on a sample of tokens of step `step`; the expert weights
    it needs are generated before the clock starts."""
    from moe_inputs import native
    from oracle import moe_oracle as mo
    h = np.stack([mi.gen_h(w, step, slice(int(t), int(t) + 1))[0] for t in tokens])
    e = mi.gen_centroids(w)
    b = mi.gen_bias(w)
    cfg = mo.LayerConfig(T=len(tokens), d_model=w.d_model, E_r=w.E_r, E_s=w.E_s, K=w.K,
                         score_fn=w.score_fn, n_groups=w.n_groups, topk_groups=w.topk_groups,
                         group_topn=w.group_topn, capacity_factor=w.capacity_factor,
                         add_residual=w.add_residual)
    s = mo.affinity(h, e, w.score_fn)
    idx = mo.select_experts(s, b, w.K, w.n_groups, w.topk_groups, w.group_topn)
    need = [(which, int(ex)) for ex in np.unique(idx) for which in ("gate", "up", "down")]
    need += [(which, j) for j in range(w.E_s) for which in ("sgate", "sup", "sdown")]
    for key in need:
        if key in _WCACHE:
            _WCACHE.move_to_end(key)
        else:
            _WCACHE[key] = native.weight_host(w, *key)
            while len(_WCACHE) > _WCACHE_MAX:
                _WCACHE.popitem(last=False)
    src = lambda which, ex: _WCACHE[(which, int(ex))]
    t0 = time.perf_counter()
    mo.layer_forward(cfg, h, e, b, src)
    return time.perf_counter() - t0


def oracle_train_sample_time(w, tokens: np.ndarray):
    """Time the oracle's layer forward + backward on a sample of tokens (the
    layer restricted to them, full-size experts; weights generated before the
    clock starts)."""
    from moe_inputs import native
    from oracle import moe_oracle as mo
    h = np.stack([mi.gen_h(w, 0, slice(int(t), int(t) + 1))[0] for t in tokens])
    e, b = mi.gen_centroids(w), mi.gen_bias(w)
    cfg = mo.LayerConfig(T=len(tokens), d_model=w.d_model, E_r=w.E_r, E_s=w.E_s, K=w.K,
                         score_fn=w.score_fn, n_groups=w.n_groups, topk_groups=w.topk_groups,
                         group_topn=w.group_topn, capacity_factor=w.capacity_factor,
                         add_residual=w.add_residual)
    s = mo.affinity(h, e, w.score_fn)
    idx = mo.select_experts(s, b, w.K, w.n_groups, w.topk_groups, w.group_topn)
    need = [(which, int(ex)) for ex in np.unique(idx) for which in ("gate", "up", "down")]
    need += [(which, j) for j in range(w.E_s) for which in ("sgate", "sup", "sdown")]
    W = {key: native.weight_host(w, *key) for key in need}
    src = lambda which, ex: W[(which, int(ex))]
    dy = np.random.default_rng(5).normal(size=h.shape)
    t0 = time.perf_counter()
    out = mo.layer_forward(cfg, h, e, b, src)
    _, gates, disp = mo.route(cfg, out["s"], b if w.score_fn == 0 else np.zeros(w.E_r, np.float32))
    mo.layer_backward(cfg, h, e, out["s"], out["idx"], gates, disp, src, dy)
    return time.perf_counter() - t0


def train_work(w, kept: np.ndarray):
    """(flops, bytes) of one backward: dA, dX and the weight gradients of every
    kept row and shared row, and the router terms; reads of every touched
    expert's weights, a write of every expert's weight gradient (zero for
    untouched ones), dy in, dh and de out."""
    n_rows = int(kept.sum())
    touched = int((kept > 0).sum())
    d, f, fs = w.d_model, w.d_ffn, w.d_ffn_shared
    flops = 12 * d * (f * n_rows + fs * w.E_s * w.T) + 4 * w.T * w.E_r * d
    nbytes = (touched * 3 * d * f * 2 + w.E_r * 3 * d * f * 2 + 2 * w.E_s * 3 * d * fs * 2
              + 3 * w.T * d * 2 + w.E_r * d * 4)
    return flops, nbytes


def train_writes(w) -> int:
    """Bytes one backward writes: every weight gradient (routed and shared,
    bf16), dh (bf16) and de (fp32)."""
    d, f, fs = w.d_model, w.d_ffn, w.d_ffn_shared
    return w.E_r * 3 * d * f * 2 + w.E_s * 3 * d * fs * 2 + w.T * d * 2 + w.E_r * d * 4


def measure_write_gbs(torch, dev, nbytes=4 << 30, reps=6) -> float:
    """HBM write-only bandwidth on this GPU now: the fastest of `reps` device
    fills of nbytes, each timed with CUDA events (a denominator for
    write-bound kernels, not our work)."""
    buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    buf.fill_(1)
    best = 0.0
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        buf.fill_(1)
        b.record()
        torch.cuda.synchronize()
        best = max(best, nbytes / (a.elapsed_time(b) * 1e-3) / 1e9)
    del buf
    return best


def run_train(args, w, rank, world, local_rank):
    """Training step: moe_layer_forward (train = 1) + moe_layer_backward."""
    import torch
    import torch.distributed as dist
    import sparse_mixture_experts_selection_b200 as moe
    from moe_inputs import native

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    W, G = {}, {}
    for k in ("gate", "up", "down", "sgate", "sup", "sdown"):
        tid, n, rows, cols, sigma = mi.weight_spec(w, k)
        if n == 0:
            W[k] = G[k] = None
            continue
        W[k] = torch.empty((n, rows, cols), dtype=torch.bfloat16, device=dev)
        native.fill_device(W[k].data_ptr(), W[k].numel(), True, w.seed, tid, 0, sigma, stream=stream.cuda_stream)
        G[k] = torch.empty_like(W[k])
    e = torch.from_numpy(mi.gen_centroids(w)).to(dev)
    b = torch.from_numpy(mi.gen_bias(w)).to(dev)
    n_steps = args.warmup + args.steps
    H = []
    for i in range(n_steps):
        t = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device=dev)
        native.fill_device(t.data_ptr(), t.numel(), True, w.seed, h_stream_id(rank, i), 0, 1.0,
                           stream=stream.cuda_stream)
        H.append(t)
    dy = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device=dev)
    native.fill_device(dy.data_ptr(), dy.numel(), True, w.seed, 77, 0, 1.0, stream=stream.cuda_stream)
    cfg = moe.config_for(w, train=1)
    ws = moe.alloc_workspace(moe.moe_workspace_size(cfg), dev)
    y = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device=dev)
    s_out = torch.empty((w.T, w.E_r), dtype=torch.float32, device=dev)
    idx = torch.empty((w.T, w.K), dtype=torch.int32, device=dev)
    kept = torch.zeros((n_steps, w.E_r), dtype=torch.int32, device=dev)
    dh = torch.empty_like(y)
    de = torch.empty((w.E_r, w.d_model), dtype=torch.float32, device=dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_steps)]

    def step(i):
        ev[i][0].record()
        moe.moe_layer_forward(cfg, H[i], e, b, W["gate"], W["up"], W["down"], W["sgate"], W["sup"],
                              W["sdown"], y, ws, idx_out=idx, kept_out=kept[i], s_out=s_out,
                              update_bias=w.gamma > 0, gamma=w.gamma)
        ev[i][1].record()
        moe.moe_layer_backward(cfg, H[i], e, s_out, idx, W["gate"], W["up"], W["down"], W["sgate"],
                               W["sup"], W["sdown"], dy, dh, de, G["gate"], G["up"], G["down"],
                               G["sgate"], G["sup"], G["sdown"], ws)
        ev[i][2].record()

    clocks = ClockSampler(torch.cuda.current_device())
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.time()
    t0.record()
    for j in range(args.steps):
        step(args.warmup + j)
    t1.record()
    torch.cuda.synchronize()
    clocks.mark(wall0, time.time())
    if world > 1:
        dist.barrier()
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), dev)
    err = moe.moe_get_device_error(ws)
    if err:
        raise RuntimeError(f"device error word {err} after the timed region")
    fwd = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.warmup, n_steps)]
    bwd = [ev[i][1].elapsed_time(ev[i][2]) for i in range(args.warmup, n_steps)]
    kept_h = kept.cpu().numpy()[args.warmup:]
    clk = clocks.summary()
    clocks.stop()
    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    hbm, bf16_peak = float(peaks["hbm_gbs"]), float(peaks["bf16_tflops"])
    tw = [train_work(w, k) for k in kept_h]
    b_flops, b_bytes = float(np.mean([x[0] for x in tw])), float(np.mean([x[1] for x in tw]))
    bwd_s = float(np.mean(bwd)) / 1000
    t_roof_b = max(b_flops / (bf16_peak * 1e12), b_bytes / (hbm * 1e9))
    # the weight-gradient launches only write (their operands are L2-resident):
    # they are bounded by the write-only bandwidth, which is well below the copy figure
    write_gbs = measure_write_gbs(torch, dev)
    b_writes = float(train_writes(w))
    t_roof_w = max(b_flops / (bf16_peak * 1e12), (b_bytes - b_writes) / (hbm * 1e9) + b_writes / (write_gbs * 1e9))
    ms_per_step = elapsed_ms / args.steps
    line = {
        "metric": "MoE-layer training step (forward + backward) tokens/s", "value": job_throughput(world, w.T, args.steps, elapsed_ms),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w), step="moe_layer_forward (train) + moe_layer_backward",
                       parallelism=f"replicas x{world}"),
        "forward_ms": float(np.mean(fwd)), "backward_ms": float(np.mean(bwd)),
        "backward_roofline": {"t_roof_ms": 1000 * t_roof_b, "frac": 1000 * t_roof_b / float(np.mean(bwd)),
                              "flops": b_flops, "bytes": b_bytes,
                              "bound": "hbm" if b_bytes / (hbm * 1e9) >= b_flops / (bf16_peak * 1e12) else "tensor",
                              "achieved_gbs": b_bytes / bwd_s / 1e9, "achieved_tflops": b_flops / bwd_s / 1e12,
                              "peaks": f"{peak_kind}: {hbm} GB/s, {bf16_peak} TFLOP/s burst",
                              "write_aware": {"t_roof_ms": 1000 * t_roof_w, "frac": 1000 * t_roof_w / float(np.mean(bwd)),
                                              "writes": b_writes, "write_gbs": write_gbs,
                                              "note": "writes at the write-only bandwidth measured live "
                                                      "(device fill), reads at the copy figure"}},
        "clocks": clk,
        # forward 11 + backward: groups, (sigmoid: scan + scatter of every selected
        # pair), 2 tail zeroings, rows, 5 GEMMs, gates, dh, de
        "gpu_launches": (11 + 12 + (2 if w.score_fn == 0 else 0)) * args.steps,
    }
    if not args.no_cpu_baseline:
        n_tok = 2
        rng = np.random.default_rng(12345)
        tokens = np.sort(rng.choice(w.T, size=n_tok, replace=False))
        dt = oracle_train_sample_time(w, tokens)
        line["cpu_baseline"] = {"value": n_tok / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{n_tok} seeded tokens: layer forward + backward restricted to "
                                          f"them, full-size experts, float64 numpy"}
    print(json.dumps(line), flush=True)


def cpu_baseline(w, n_tokens: int):
    rng = np.random.default_rng(12345)
    tokens = np.sort(rng.choice(w.T, size=n_tokens, replace=False))
    dt = oracle_sample_time(w, tokens)
    return {"value": n_tokens / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n_tokens} of the {w.T} tokens of one batch (seeded sample), full layer "
                      f"forward on them in float64 numpy; weight generation excluded",
            "seconds": dt}


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    per_step = args.ref_tokens
    times = []
    for i in range(args.warmup + args.steps):
        rng = np.random.default_rng(1000 + i)
        tokens = np.sort(rng.choice(w.T, size=per_step, replace=False))
        dt = oracle_sample_time(w, tokens, step=i % max(1, w.steps))
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = per_step * len(times) / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000 * total / len(times), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(workload_config(w), parallelism=f"replicas x{world}"),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": f"each step: {per_step} seeded tokens of the batch, full layer "
                                       f"forward in float64 numpy"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(w):
    return {"workload": w.name, "T": w.T, "d_model": w.d_model, "E_r": w.E_r, "E_s": w.E_s, "K": w.K,
            "d_ffn": w.d_ffn, "d_ffn_shared": w.d_ffn_shared,
            "routing": "sigmoid, bias-only selection" if w.score_fn == 0 else "softmax",
            "groups": f"{w.n_groups} groups, keep {w.topk_groups}, group score = top-{w.group_topn} sum"
            if w.n_groups > 1 else "none",
            "bias_step": f"gamma={w.gamma} every step" if w.gamma else "none",
            "capacity_factor": w.capacity_factor,
            "l2": "inputs larger than L2 (expert weights stream from HBM every step)"}


# ---------------------------------------------------------------------------
# replicas (N > 1): one process per GPU, no data-path collective
# ---------------------------------------------------------------------------

def h_stream_id(rank: int, step: int) -> int:
    """Tensor id of the token batch of `step` on replica `rank` (distinct per rank)."""
    return mi.h_tensor_id(rank * 100000 + step)


def max_over_ranks(x: float, device=None) -> float:
    """The max of a per-rank float over all ranks (timing only)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_step: int, steps: int, max_ms: float) -> float:
    """Whole-job tokens/s: every replica's tokens over the slowest replica's time."""
    return world * tokens_per_step * steps / (max_ms / 1000.0)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def make_inputs(w, dev, stream, rank, n_steps, moe, native):
    """Device-resident inputs of a workload: weights (e4m3 blobs for the
    e4m3-weight layers), centroids, bias and one fresh token batch per step."""
    import torch
    bf16 = w.dtype != "f32"                 # bf16 activations (bf16 and e4m3-weight layers)
    e4m3 = w.dtype == "bf16_e4m3"
    dt = torch.bfloat16 if bf16 else torch.float32
    W = {}
    for k in ("gate", "up", "down", "sgate", "sup", "sdown"):
        tid, n, rows, cols, sigma = mi.weight_spec(w, k)
        if n == 0:
            W[k] = None
            continue
        t = torch.empty((n, rows, cols), dtype=dt, device=dev)
        native.fill_device(t.data_ptr(), t.numel(), bf16, w.seed, tid, 0, sigma, stream=stream.cuda_stream)
        if e4m3:
            # the same bf16 weights as e4m3 blobs (codes + row scales); the bf16 copy is dropped
            q = torch.empty(moe.moe_quantized_bytes(n * rows, cols), dtype=torch.uint8, device=dev)
            moe.moe_quantize_rows(t, moe.DTYPE_BF16, n * rows, cols, q, stream=stream)
            stream.synchronize()
            del t
            t = q
        W[k] = t
    e = torch.from_numpy(mi.gen_centroids(w)).to(dev)
    b = torch.from_numpy(mi.gen_bias(w)).to(dev)
    H = []
    for i in range(n_steps):
        t = torch.empty((w.T, w.d_model), dtype=dt, device=dev)
        native.fill_device(t.data_ptr(), t.numel(), bf16, w.seed, h_stream_id(rank, i), 0, 1.0,
                           stream=stream.cuda_stream)
        H.append(t)
    return {"W": W, "e": e, "b": b, "H": H, "dt": dt}


class LayerRun:
    """moe_layer_forward (with the bias step when the workload has one) over
    the workload's fresh batches, with phase events and per-step loads."""

    def __init__(self, w, inp, dev, moe, n_steps):
        import torch
        self.w, self.inp, self.moe = w, inp, moe
        self.cfg = moe.config_for(w)
        self.ws = moe.alloc_workspace(moe.moe_workspace_size(self.cfg), dev)
        self.y = torch.empty((w.T, w.d_model), dtype=inp["dt"], device=dev)
        self.kept = torch.zeros((n_steps, w.E_r), dtype=torch.int32, device=dev)
        self.counts = torch.zeros((n_steps, w.E_r), dtype=torch.int32, device=dev)
        self.max_vio = torch.zeros(n_steps, dtype=torch.float32, device=dev)

    def step(self, i, hh=None, yy=None):
        W, inp, w = self.inp["W"], self.inp, self.w
        self.moe.moe_layer_forward(self.cfg, inp["H"][i] if hh is None else hh, inp["e"], inp["b"], W["gate"],
                                   W["up"], W["down"], W["sgate"], W["sup"], W["sdown"],
                                   self.y if yy is None else yy, self.ws, counts_out=self.counts[i],
                                   kept_out=self.kept[i], update_bias=w.gamma > 0, gamma=w.gamma,
                                   max_vio_out=self.max_vio[i:i + 1])

    def timed(self, first, steps, world, dev, clocks=None):
        """Time steps first .. first+steps-1 (CUDA events on the launch stream,
        barrier + synchronize on both sides, max over ranks); returns
        (elapsed_ms, phase_ms [steps, phases], clock summary)."""
        import torch
        import torch.distributed as dist
        moe = self.moe
        n_ph = len(moe.PHASES) + 1
        ph_events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ph)] for _ in range(steps)]
        for evs in ph_events:
            for ev in evs:
                ev.record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        wall0 = time.time()
        t_start.record()
        for j in range(steps):
            moe.moe_set_phase_events(ph_events[j])
            self.step(first + j)
        t_end.record()
        torch.cuda.synchronize()
        wall1 = time.time()
        moe.moe_set_phase_events([])
        if world > 1:
            dist.barrier()
        elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
        err = moe.moe_get_device_error(self.ws)
        if err:
            raise RuntimeError(f"device error word {err} after the timed region")
        phase_ms = np.array([[evs[i].elapsed_time(evs[i + 1]) for i in range(n_ph - 1)] for evs in ph_events])
        clk = clocks.summary((wall0, wall1)) if clocks else None
        return elapsed_ms, phase_ms, clk


def kernel_records(w, kept_h, phase_ms, ms_per_step, moe):
    """Roofline records of the step and of its two grouped GEMMs (the gate/up
    GEMM is the dominant kernel), by the roofline definition's bytes and
    FLOPs, against the measured peaks (burst GEMM figure: the timed regions
    last well under a second)."""
    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    e4m3 = w.dtype == "bf16_e4m3"
    # e4m3 tensor-core peak: the measured bf16 figure x the nominal fp8/bf16 ratio (4.5 / 2.25)
    mma_peak = float(peaks["bf16_tflops"]) * (2.0 if e4m3 else 1.0)
    peak_note = f"{peak_kind}: {hbm} GB/s, {mma_peak} TFLOP/s burst" + (" (e4m3: bf16 x 2, nominal ratio)" if e4m3 else "")
    gu_s = float(np.mean(phase_ms[:, moe.PHASES.index("ffn_gate_up")])) / 1000.0
    dn_s = float(np.mean(phase_ms[:, moe.PHASES.index("ffn_down")])) / 1000.0
    mean = lambda f: tuple(float(np.mean([f(w, k)[i] for k in kept_h])) for i in range(2))
    gu_flops, gu_bytes = mean(gateup_work)
    dn_flops, dn_bytes = mean(down_work)
    l_flops, l_bytes = mean(layer_work)
    gu_impl = float(np.mean([gateup_impl_bytes(w, k) for k in kept_h]))
    t_roof = max(l_flops / (mma_peak * 1e12), l_bytes / (hbm * 1e9))
    gu = {"bound": "hbm" if gu_bytes / (hbm * 1e9) >= gu_flops / (mma_peak * 1e12) else "tensor",
          "achieved_gbs": gu_bytes / gu_s / 1e9, "frac_hbm": gu_bytes / gu_s / 1e9 / hbm,
          "achieved_tflops": gu_flops / gu_s / 1e12, "frac_tensor": gu_flops / gu_s / 1e12 / mma_peak,
          "ms": 1000 * gu_s, "bytes": gu_bytes, "flops": gu_flops,
          "impl_bytes": gu_impl, "kernel_traffic_frac": gu_impl / gu_s / 1e9 / hbm}
    dn = {"achieved_gbs": dn_bytes / dn_s / 1e9, "frac_hbm": dn_bytes / dn_s / 1e9 / hbm,
          "achieved_tflops": dn_flops / dn_s / 1e12, "frac_tensor": dn_flops / dn_s / 1e12 / mma_peak,
          "ms": 1000 * dn_s, "bytes": dn_bytes, "flops": dn_flops}
    layer = {"t_roof_ms": 1000 * t_roof, "frac": 1000 * t_roof / ms_per_step, "flops": l_flops, "bytes": l_bytes,
             "bound": "hbm" if l_bytes / (hbm * 1e9) >= l_flops / (mma_peak * 1e12) else "tensor",
             "frac_hbm": l_bytes / (hbm * 1e9) * 1000 / ms_per_step,
             "frac_tensor": l_flops / (mma_peak * 1e12) * 1000 / ms_per_step, "peaks": peak_note}
    return gu, dn, layer, hbm, mma_peak, peak_kind


def gemm_tile_rows(w, moe) -> int:
    """Row-tile height of the layer's grouped GEMMs as the library chooses it:
    256 on CTA pairs, 128 single-CTA tensor-core, the CUDA-core tile for fp32
    (the layer provisions min(T*K, E_r * capacity) routed rows)."""
    rows = w.T * w.K
    if w.capacity_factor > 0:
        rows = min(rows, w.E_r * int(math.floor(w.T * w.K * w.capacity_factor / w.E_r)))
    return moe.moe_expert_ffn_tile_rows(moe.config_for(w), w.E_r, max(rows, 1))


def launches_per_step(w) -> int:
    """Our kernels per layer step: [centroid split + router GEMM | CUDA-core
    logits], select, scan, scatter, row gather (e4m3: quantize h + gather),
    group tables, gate/up GEMM, down GEMM, combine, bias step; e4m3 adds the
    quantization of A (and of the shared A when there are shared experts)."""
    bf16 = w.dtype != "f32"
    e4m3 = w.dtype == "bf16_e4m3"
    return (11 if bf16 else 10) + ((1 + 2 * (w.E_s > 0)) if e4m3 else 0)


def measure_extra(name, args, rank, world, dev, stream, moe, native, clocks):
    """One sub-record: a workload timed alone on this GPU (at least ~200 ms of
    timed steps so that the clock samples cover it)."""
    import torch
    w = mi.WORKLOADS[name]
    warm = args.warmup
    probe = make_inputs(w, dev, stream, rank, warm, moe, native)
    run = LayerRun(w, probe, dev, moe, warm)
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(warm):
        run.step(i)
    b_.record()
    torch.cuda.synchronize()
    est_ms = a.elapsed_time(b_) / warm
    steps = int(min(4000, max(args.steps, math.ceil(200.0 / max(est_ms, 1e-3)))))
    del run
    # fresh batches for warm-up + timed steps; the weights of the probe are reused
    H = []
    for i in range(warm + steps):
        t = torch.empty((w.T, w.d_model), dtype=probe["dt"], device=dev)
        native.fill_device(t.data_ptr(), t.numel(), w.dtype != "f32", w.seed, h_stream_id(rank, i), 0, 1.0,
                           stream=stream.cuda_stream)
        H.append(t)
    inp = dict(probe, H=H, b=torch.from_numpy(mi.gen_bias(w)).to(dev))
    run = LayerRun(w, inp, dev, moe, warm + steps)
    for i in range(warm):
        run.step(i)
    torch.cuda.synchronize()
    elapsed_ms, phase_ms, clk = run.timed(warm, steps, world, dev, clocks)
    ms = elapsed_ms / steps
    kept_h = run.kept.cpu().numpy()[warm:]
    counts_h = run.counts.cpu().numpy()[warm:]
    gu, dn, layer, _, _, _ = kernel_records(w, kept_h, phase_ms, ms, moe)
    gu["tile_rows"] = dn["tile_rows"] = gemm_tile_rows(w, moe)
    rec = {"value": job_throughput(world, w.T, steps, elapsed_ms), "unit": "tokens/s", "ms_per_step": ms,
           "steps": steps, "warmup": warm, "dtype": {"bf16": "bf16", "bf16_e4m3": "e4m3"}.get(w.dtype, "f32"),
           "config": workload_config(w), "layer_roofline": layer, "gate_up_gemm": gu, "down_gemm": dn,
           "phases_ms": {p: float(np.mean(phase_ms[:, i])) for i, p in enumerate(moe.PHASES)},
           "rows_per_step": float(np.mean(kept_h.sum(1))), "touched_experts": float(np.mean((kept_h > 0).sum(1))),
           "dropped_pairs_per_step": float(np.mean(counts_h.sum(1) - kept_h.sum(1))),
           "clocks": clk, "gpu_launches": launches_per_step(w) * steps}
    if w.gamma > 0:
        vio = run.max_vio.cpu().numpy()[warm:]
        rec["max_vio_first_last"] = [round(float(vio[0]), 4), round(float(vio[-1]), 4)]
    del run, inp, probe, H
    torch.cuda.empty_cache()
    return rec


EXTRA_WORKLOADS = ["deepseek_v3_decode", "mixtral_8x14336", "finegrained_64x1408", "finegrained_64x1408_cf1.25",
                   "toy_fp32"]


def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import sparse_mixture_experts_selection_b200 as moe
    from moe_inputs import native

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    bf16 = w.dtype != "f32"
    e4m3 = w.dtype == "bf16_e4m3"
    dt = torch.bfloat16 if bf16 else torch.float32
    clocks = ClockSampler(torch.cuda.current_device())

    # ---- inputs resident in HBM ----
    n_steps = args.warmup + args.steps
    inp = make_inputs(w, dev, stream, rank, n_steps, moe, native)
    run = LayerRun(w, inp, dev, moe, n_steps)
    for i in range(args.warmup):
        run.step(i)
    torch.cuda.synchronize()
    b_after_warmup = inp["b"].clone()
    elapsed_ms, phase_ms, clk = run.timed(args.warmup, args.steps, world, dev, clocks)
    kept_h = run.kept.cpu().numpy()[args.warmup:]
    vio_h = run.max_vio.cpu().numpy()
    value = job_throughput(world, w.T, args.steps, elapsed_ms)
    ms_per_step = elapsed_ms / args.steps

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        # Public API end to end: pinned host h in, layer, y back to pinned host,
        # every step.  Copies run on a second stream, double-buffered, so the
        # H2D of step j+1 and the D2H of step j overlap the compute of the
        # neighbouring steps; the timed region spans the first H2D to the last D2H.
        H = inp["H"]
        pin_h = [H[i].cpu().pin_memory() for i in range(args.warmup, n_steps)]
        y_host = [torch.empty((w.T, w.d_model), dtype=dt).pin_memory() for _ in range(2)]
        h_dev = [torch.empty_like(H[0]) for _ in range(2)]
        y_dev = [run.y, torch.empty_like(run.y)]
        inp["b"].copy_(b_after_warmup)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        main, cs = torch.cuda.current_stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        h_ready = [ev() for _ in range(args.steps)]
        done = [ev() for _ in range(args.steps)]
        y_read = [ev() for _ in range(args.steps)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        cs.wait_event(e0)
        with torch.cuda.stream(cs):
            h_dev[0].copy_(pin_h[0], non_blocking=True)
            h_ready[0].record(cs)
        for j in range(args.steps):
            buf = j % 2
            main.wait_event(h_ready[j])
            if j >= 2:
                main.wait_event(y_read[j - 2])          # y_dev[buf] has been read back
            run.step(args.warmup + j, h_dev[buf], y_dev[buf])
            done[j].record(main)
            with torch.cuda.stream(cs):
                if j + 1 < args.steps:
                    if j >= 1:
                        cs.wait_event(done[j - 1])      # h_dev[(j+1)%2] no longer in use
                    h_dev[(j + 1) % 2].copy_(pin_h[j + 1], non_blocking=True)
                    h_ready[j + 1].record(cs)
                cs.wait_event(done[j])
                y_host[buf].copy_(y_dev[buf], non_blocking=True)
                y_read[j].record(cs)
        main.wait_event(y_read[args.steps - 1])
        e1.record(main)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        es = 2 if bf16 else 4
        e2e = {"value": job_throughput(world, w.T, args.steps, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": w.T * w.d_model * es, "d2h_bytes_per_step": w.T * w.d_model * es,
               "copies": "pinned host, second stream, double-buffered"}
        del pin_h, y_host, h_dev, y_dev

    gu, dn, layer, hbm, mma_peak, peak_kind = kernel_records(w, kept_h, phase_ms, ms_per_step, moe)
    gu["tile_rows"] = dn["tile_rows"] = gemm_tile_rows(w, moe)
    # DRAM traffic per launch: the ncu capture's DRAM bytes over its implementation
    # bytes (profiles/traffic.json), scaled to this launch's implementation bytes
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            doc = json.load(f)
        rec = doc.get("ffn_gate_up")
        src = os.path.join(ROOT, doc.get("source", ""))
        # counters taken on another version of the kernel say nothing about this one
        same = os.path.isfile(src) and hashlib.sha256(open(src, "rb").read()).hexdigest() == doc.get("source_sha256")
        if rec and same and w.dtype == "bf16":       # counters of the bf16 kernel
            traffic = rec["ratio"] * gu["impl_bytes"]
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if e4m3 else ("bf16" if bf16 else "f32"),
        "data": "synthetic", "config": dict(workload_config(w), parallelism=f"replicas x{world}"),
        "roofline": {"bound": "hbm", "achieved": gu["achieved_gbs"], "peak": hbm, "unit": "GB/s",
                     "frac": gu["frac_hbm"], "traffic": traffic,
                     "kernel": "ffn_gate_up (tcgen05 grouped GEMM)",
                     "bytes_per_launch": gu["bytes"],
                     "bytes_def": "touched routed gate+up weights + shared gate+up weights + h read once",
                     "peak_source": f"{peak_kind} hbm_gbs (of {peak_kind})",
                     "kernel_traffic_frac": gu["kernel_traffic_frac"],
                     "kernel_traffic_note": "implementation bytes (adds the permuted-row read and the "
                                            "SwiGLU-product write) over the same time",
                     "tensor_tflops": gu["achieved_tflops"], "tensor_frac_burst": gu["frac_tensor"]},
        "layer_roofline": layer,
        "phases_ms": {p: float(np.mean(phase_ms[:, i])) for i, p in enumerate(moe.PHASES)},
        "down_gemm": dn,
        "rows_per_step": float(np.mean(kept_h.sum(1))),
        "touched_experts": float(np.mean((kept_h > 0).sum(1))),
        "max_vio": [round(float(v), 4) for v in vio_h[args.warmup:]],
        "e2e": e2e,
        "clocks": clk,
        "gpu_launches": launches_per_step(w) * args.steps,
    }
    del run, inp
    torch.cuda.empty_cache()
    if world == 1 and args.workloads != "none":
        names = EXTRA_WORKLOADS if args.workloads == "all" else [n for n in args.workloads.split(",") if n]
        line["workloads"] = {n: measure_extra(n, args, rank, world, dev, stream, moe, native, clocks)
                             for n in names if n != w.name}
    clocks.stop()
    if rank != 0:
        return
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_tokens)
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(mi.WORKLOADS))
    ap.add_argument("--cpu-tokens", type=int, default=8, help="tokens in the cpu_baseline sample")
    ap.add_argument("--ref-tokens", type=int, default=2, help="tokens per --impl reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--workloads", default="all",
                    help="sub-records of the N=1 line: 'all' (the other configurations), 'none', or a "
                         "comma-separated list of workload names")
    ap.add_argument("--train", action="store_true",
                    help="time the training step (forward with train = 1 + moe_layer_backward)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="profiling only: tokens per step (with --experts)")
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling only: run the workload with this many routed experts (smaller "
                         "device footprint for ncu captures); not a bench configuration")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = mi.WORKLOADS[args.workload]
    if args.experts:
        w = w.with_(name=f"{w.name}_E{args.experts}", E_r=args.experts,
                    n_groups=min(w.n_groups, args.experts // 4) if w.n_groups > 1 else 1)
    if args.tokens:
        w = w.with_(name=f"{w.name}_T{args.tokens}", T=args.tokens)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.train:
            run_train(args, w, rank, world, local_rank)
        else:
            run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

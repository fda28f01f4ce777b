"""A model of where the training path stores bf16 values, used to derive the
tolerance of the backward parity tests (test infrastructure, never the product
path).

The layer's GPU backward multiplies bf16 operands with fp32 accumulation and
keeps these intermediates in bf16: the forward's U, V and A = SiLU(U) V; in
the backward g*dy (dO), dU, dV, each expert's dX, the weight gradients and dh
-- and the gate-scaled expert output (slot) in fp16.  This model repeats the
exact float64 arithmetic of the oracle's layer backward with a round to bf16
(fp16 for the slot) at exactly those points, and nowhere else.  Its distance from the oracle is the
error those roundings alone cause; the parity bar must sit above it.
"""
import numpy as np

import moe_inputs as mi
from oracle import moe_oracle as mo


def _rb(a):
    return mi.round_bf16(np.asarray(a, np.float32)).astype(np.float64)


def _rh(a):
    return np.asarray(a, np.float32).astype(np.float16).astype(np.float64)


def _expert(x, wg, wu, wd, g, dy):
    x = np.asarray(x, np.float64)
    wg, wu, wd = (np.asarray(w, np.float64) for w in (wg, wu, wd))
    u, v = x @ wg.T, x @ wu.T
    a = _rb(u / (1.0 + np.exp(-u)) * v)
    slot = _rh(g * (a @ wd.T))
    ub, vb = _rb(u), _rb(v)
    sig = 1.0 / (1.0 + np.exp(-ub))
    do = _rb(g * dy)
    da = do @ wd
    du = _rb(da * vb * sig * (1.0 + ub * (1.0 - sig)))
    dv = _rb(da * ub * sig)
    dx = _rb(du @ wg + dv @ wu)
    dg = (dy * slot).sum(axis=1) / g[:, 0]
    return dx, _rb(du.T @ x), _rb(dv.T @ x), _rb(do.T @ a), dg


def layer_backward_bf16(cfg, h, e, s32, idx, gates, disp, weights, dy):
    """Same inputs and outputs as the oracle's layer_backward."""
    x = np.asarray(h, np.float64)
    dy = np.asarray(dy, np.float64)
    dh = dy * float(cfg.add_residual)
    grads = {}
    ones = np.ones((cfg.T, 1))
    for j in range(cfg.E_s):
        dx, dwg, dwu, dwd, _ = _expert(x, weights("sgate", j), weights("sup", j), weights("sdown", j), ones, dy)
        dh = dh + dx
        grads[("sgate", j)], grads[("sup", j)], grads[("sdown", j)] = dwg, dwu, dwd
    dg = np.zeros((cfg.T, cfg.K))
    kept = disp.row_of >= 0
    ex_of = idx.astype(np.int64)
    for ex in np.unique(ex_of[kept]):
        rows, ks = np.nonzero((ex_of == ex) & kept)
        g = gates[rows, ks].astype(np.float64)[:, None]
        dx, dwg, dwu, dwd, dgv = _expert(x[rows], weights("gate", ex), weights("up", ex), weights("down", ex),
                                         g, dy[rows])
        np.add.at(dh, rows, dx)
        dg[rows, ks] = dgv
        grads[("gate", ex)], grads[("up", ex)], grads[("down", ex)] = dwg, dwu, dwd
    dz = mo.score_backward(s32, mo.gate_backward(s32, idx, dg), cfg.score_fn)
    dh = dh + dz @ np.asarray(e, np.float64)
    return dict(dh=_rb(dh), de=dz.T @ x, dz=dz, grads=grads)

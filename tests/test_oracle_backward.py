"""Pins of the oracle's layer backward: torch.autograd (float64) through a
dense restatement of the forward with the routing held fixed -- an
independent differentiation of the same definition -- plus finite
differences and the structural facts (the bias gets no gradient, unselected
experts get none, dropped pairs give dg = 0)."""
import numpy as np
import torch

from oracle import moe_oracle as mo

F32 = np.float32


def _case(score_fn, E_s, cf, seed, T=24, d=16, E=8, K=2, f=12, fs=10):
    rng = np.random.default_rng(seed)
    h = rng.normal(size=(T, d))
    e = rng.normal(size=(E, d)).astype(F32) * 0.5
    b = (rng.uniform(-0.05, 0.05, E) if score_fn == 0 else np.zeros(E)).astype(F32)
    W = {k: rng.normal(size=(E, f, d)) / np.sqrt(d) for k in ("gate", "up")}
    W["down"] = rng.normal(size=(E, d, f)) / np.sqrt(f)
    W.update({k: rng.normal(size=(max(E_s, 1), fs, d)) / np.sqrt(d) for k in ("sgate", "sup")})
    W["sdown"] = rng.normal(size=(max(E_s, 1), d, fs)) / np.sqrt(fs)
    cfg = mo.LayerConfig(T=T, d_model=d, E_r=E, E_s=E_s, K=K, score_fn=score_fn, capacity_factor=cf)
    s = mo.affinity(h, e, score_fn)
    idx, gates, disp = mo.route(cfg, s, b)
    dy = rng.normal(size=(T, d))
    src = lambda which, ex: W[which][ex]
    return cfg, h, e, b, W, s, idx, gates, disp, dy, src


def _torch_grads(cfg, h, e, W, idx, disp, dy):
    """Autograd of y = a h + sum_j shared_j(h) + sum_{k kept} g_k expert_{I_k}(h),
    g from the (sigmoid / softmax) scores of z = h e^T renormalised over I_t."""
    th = torch.tensor(h, dtype=torch.float64, requires_grad=True)
    te = torch.tensor(e.astype(np.float64), requires_grad=True)
    tW = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in W.items()}
    z = th @ te.T
    s = torch.sigmoid(z) if cfg.score_fn == 0 else torch.softmax(z, dim=-1)
    ti = torch.tensor(idx.astype(np.int64))
    sel = torch.gather(s, 1, ti)
    g = sel / torch.clamp(sel.sum(dim=1, keepdim=True), min=1e-12)
    silu = torch.nn.functional.silu
    y = th * cfg.add_residual
    for j in range(cfg.E_s):
        y = y + (silu(th @ tW["sgate"][j].T) * (th @ tW["sup"][j].T)) @ tW["sdown"][j].T
    for t in range(cfg.T):
        for k in range(cfg.K):
            if disp.row_of[t, k] < 0:
                continue
            ex = int(idx[t, k])
            o = (silu(th[t] @ tW["gate"][ex].T) * (th[t] @ tW["up"][ex].T)) @ tW["down"][ex].T
            y = y.index_add(0, torch.tensor([t]), (g[t, k] * o)[None])
    (y * torch.tensor(dy)).sum().backward()
    return th.grad.numpy(), te.grad.numpy(), {
        k: (v.grad.numpy() if v.grad is not None else np.zeros(v.shape)) for k, v in tW.items()}


def _check(score_fn, E_s, cf, seed):
    cfg, h, e, b, W, s, idx, gates, disp, dy, src = _case(score_fn, E_s, cf, seed)
    out = mo.layer_backward(cfg, h, e, s, idx, gates, disp, src, dy)
    dh, de, gW = _torch_grads(cfg, h, e, W, idx, disp, dy)
    # the oracle's scores and gates are fp32 values (the method's own precision),
    # torch's are exact: every gradient that passes through them differs by
    # O(1e-7) relative; a wrong term or index would differ by O(1)
    close = lambda a, b, tol: np.max(np.abs(a - b)) <= tol * np.max(np.abs(b))   # normwise
    assert close(out["dh"], dh, 1e-6)
    assert close(out["de"], de, 1e-5)
    for (which, ex), g in out["grads"].items():
        assert close(g, gW[which][ex], 1e-6), (which, ex)
    used = {(w_, ex) for (w_, ex) in out["grads"]}
    for which in ("gate", "up", "down"):
        for ex in range(cfg.E_r):
            if (which, ex) not in used:
                assert np.all(gW[which][ex] == 0)          # unselected / fully dropped experts
    return out


def test_backward_sigmoid_with_shared_matches_autograd():
    _check(score_fn=0, E_s=1, cf=0.0, seed=0)


def test_backward_softmax_matches_autograd():
    _check(score_fn=1, E_s=0, cf=0.0, seed=1)


def test_backward_with_capacity_drops_matches_autograd():
    out = _check(score_fn=0, E_s=2, cf=0.5, seed=2)
    assert np.any(out["dg"] == 0)                          # dropped pairs carry no gate gradient


def test_bias_gets_no_gradient_and_dh_by_finite_differences():
    cfg, h, e, b, W, s, idx, gates, disp, dy, src = _case(0, 1, 0.0, 3)
    out = mo.layer_backward(cfg, h, e, s, idx, gates, disp, src, dy)

    def loss(hh, bb):
        ss = mo.affinity(hh, e, 0)
        ii, gg, dd = mo.route(cfg, ss, bb)
        assert np.array_equal(ii, idx)                      # small steps keep the routing
        return float((mo.layer_output(cfg, hh, ii, gg, dd, src) * dy).sum())

    # the bias moves the selection only: a nudge that keeps I_t changes nothing
    assert loss(h, b + np.float32(1e-4)) == loss(h, b)
    rng = np.random.default_rng(9)
    for _ in range(3):
        t, c = rng.integers(cfg.T), rng.integers(cfg.d_model)
        hp, hm = h.copy(), h.copy()
        hp[t, c] += 1e-4
        hm[t, c] -= 1e-4
        fd = (loss(hp, b) - loss(hm, b)) / 2e-4
        # the scores are rounded to fp32, so the difference quotient carries ~1e-7/1e-4 noise
        assert abs(fd - out["dh"][t, c]) <= 2e-3 * max(1.0, abs(fd))


def test_planted_mistakes_are_caught(monkeypatch):
    """Each plausible slip in the backward fails the autograd comparison."""
    import pytest
    good_swiglu, good_gate = mo.swiglu_backward, mo.gate_backward

    def silu_prime_without_product_term(x, wg, wu, wd, do):
        x = np.asarray(x, np.float64)
        u, v = x @ wg.T, x @ wu.T
        sig = 1 / (1 + np.exp(-u))
        a = u * sig * v
        da = do @ wd
        du, dv = da * v * sig, da * u * sig                # drops sig * u * (1 - sig)
        return du @ wg + dv @ wu, du.T @ x, dv.T @ x, do.T @ a, a @ wd.T

    def gate_without_normalisation_term(s32, idx, dg):
        s = np.asarray(s32, np.float64)
        S = np.take_along_axis(s, idx.astype(np.int64), 1).sum(1)
        ds = np.zeros_like(s)
        np.put_along_axis(ds, idx.astype(np.int64), dg / S[:, None], 1)
        return ds

    for name, fake in (("swiglu_backward", silu_prime_without_product_term),
                       ("gate_backward", gate_without_normalisation_term)):
        monkeypatch.setattr(mo, name, fake)
        with pytest.raises(AssertionError):
            _check(score_fn=0, E_s=1, cf=0.0, seed=0)
        monkeypatch.setattr(mo, "swiglu_backward", good_swiglu)
        monkeypatch.setattr(mo, "gate_backward", good_gate)

"""Pins of the oracle's router losses and logging statistics to the facts the
pages state about them and to closed forms."""
import math

import numpy as np
import torch

from oracle import moe_oracle as mo

F32 = np.float32


def _uniform_routing(T, E, K):
    # token t picks experts (t*K .. t*K+K-1) mod E: every expert is picked T*K/E times
    return np.array([[(t * K + k) % E for k in range(K)] for t in range(T)], dtype=np.int32)


def test_aux_loss_minimum_is_alpha_at_uniform_load():
    """The Switch balance term sum_i f_i P_i takes its minimum, 1, at a uniform
    load and uniform mean scores ("Sparse Mixture-of-Experts ...", section 1);
    the f_i always add up to E_r."""
    T, E, K = 64, 8, 2
    idx = np.sort(_uniform_routing(T, E, K), axis=1)
    s = np.full((T, E), 0.5, F32)                     # P_i = 1/E_r
    assert mo.aux_loss(s, idx, E, K, alpha=1.0) == 1.0
    f = E / (K * T) * mo.load_counts(idx, E)
    assert f.sum() == E
    # any other load with the same P gives the same value (f sums to E_r); a
    # skewed P aligned with a skewed load gives more
    rng = np.random.default_rng(0)
    z = rng.normal(size=(T, E)).astype(F32)
    s2 = mo.sigmoid_scores(z)
    idx2 = mo.select_experts(s2, np.zeros(E, F32), K)
    assert mo.aux_loss(s2, idx2, E, K, 1.0) > 1.0


def test_aux_loss_matches_the_pages_switch_formula_for_softmax():
    """For softmax routing P_i = mean softmax and f_i = E * one_hot.mean(0,1):
    restated with torch ops as in the ClassicalTopKRouter (section 1)."""
    rng = np.random.default_rng(1)
    T, E, K = 50, 8, 2
    z = rng.normal(size=(T, E)).astype(F32)
    p = mo.softmax_scores(z)
    idx = mo.select_experts(p, np.zeros(E, F32), K)
    one_hot = torch.nn.functional.one_hot(torch.from_numpy(idx.astype(np.int64)), E).double()
    f = one_hot.mean(dim=(0, 1)) * E
    P = torch.from_numpy(p.astype(np.float64)).mean(0)
    want = 0.01 * float((f * P).sum())
    assert math.isclose(mo.aux_loss(p, idx, E, K, 0.01), want, rel_tol=1e-6)


def test_z_loss_closed_form():
    T, E = 10, 16
    z = np.full((T, E), 3.0, F32)                     # logsumexp = 3 + log E
    assert math.isclose(mo.z_loss(z, 1e-3), 1e-3 * (3 + math.log(E)) ** 2, rel_tol=1e-12)
    rng = np.random.default_rng(2)
    z = (rng.normal(size=(T, E)) * 5).astype(F32)
    want = 1e-3 * float((torch.logsumexp(torch.from_numpy(z.astype(np.float64)), -1) ** 2).mean())
    assert math.isclose(mo.z_loss(z, 1e-3), want, rel_tol=1e-12)


def test_seq_balance_loss_reduces_to_aux_for_one_sequence():
    rng = np.random.default_rng(3)
    T, E, K = 96, 16, 4
    s = mo.sigmoid_scores(rng.normal(size=(T, E)).astype(F32))
    idx = mo.select_experts(s, np.zeros(E, F32), K)
    a = mo.aux_loss(s, idx, E, K, 1e-4)
    assert math.isclose(mo.seq_balance_loss(s, idx, E, K, T, 1e-4), a, rel_tol=1e-12)
    # two sequences: the average of the two per-sequence losses
    half = T // 2
    both = (mo.aux_loss(s[:half], idx[:half], E, K, 1e-4) + mo.aux_loss(s[half:], idx[half:], E, K, 1e-4)) / 2
    assert math.isclose(mo.seq_balance_loss(s, idx, E, K, half, 1e-4), both, rel_tol=1e-12)


def test_entropy_and_dropped_rate():
    E = 8
    assert math.isclose(mo.load_entropy(np.full(E, 5)), math.log(E), rel_tol=1e-12)
    one_hot = np.zeros(E, np.int64)
    one_hot[3] = 40
    assert mo.load_entropy(one_hot) == 0.0
    assert mo.dropped_rate(np.array([5, 4, 3, 3]), np.array([10, 4, 3, 3])) == 0.25
    assert mo.dropped_rate(np.array([1, 2]), np.array([1, 2])) == 0.0

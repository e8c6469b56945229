"""Look-ahead selection of the oracle, pinned to the optimisation it solves.

LAMP summary, "Theoretical basis": item 2 states the problem
min ||q||_0 s.t. kappa(q) <= tau; item 3 (softmax bullet) states the closed form
2 z_j (1 - z_j) |y_j| > tau for the norm-wise l1 objective (total probability
mass shift). "Experimental results": the relaxed relative-threshold variant.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle


def softmax64(y):
    y = np.asarray(y, dtype=np.float64)
    e = np.exp(y - y.max())
    return e / e.sum()


def jacobian_l1_columns_fd(y, h=1e-6):
    """l1 norm of each column of d softmax / d y by central differences (double)."""
    y = np.asarray(y, dtype=np.float64)
    n = y.size
    cols = np.zeros(n)
    for j in range(n):
        e = np.zeros(n)
        e[j] = h
        cols[j] = np.abs((softmax64(y + e) - softmax64(y - e)) / (2 * h)).sum()
    return cols


def test_criterion_is_jacobian_column_norm_times_magnitude():
    """c_j / |y_j| must be the l1 norm of the softmax Jacobian's column j: the
    first-order mass shift caused by a unit relative error in y_j."""
    rng = np.random.default_rng(0)
    for n in (2, 3, 7, 20):
        y = (rng.standard_normal(n) * 2).astype(np.float32)
        c = oracle.strict_criterion(y)
        fd = jacobian_l1_columns_fd(y)
        assert np.allclose(c / np.abs(y.astype(np.float64)), fd, rtol=1e-6, atol=1e-9)


def test_closed_form_values():
    s2 = 1.0 / (1.0 + math.exp(-2.0))   # softmax of (1, -1) and of (2, 0) is (s2, 1 - s2)
    assert np.allclose(oracle.strict_criterion(np.array([1, -1], np.float32)),
                       [2 * s2 * (1 - s2), 2 * s2 * (1 - s2)], rtol=1e-14)
    assert np.allclose(oracle.strict_criterion(np.array([2, 0], np.float32)),
                       [4 * s2 * (1 - s2), 0.0], rtol=1e-14)
    assert np.allclose(oracle.strict_criterion(np.array([1, 1, 1], np.float32)), [4 / 9] * 3, rtol=1e-14)
    # a single valid key has z = 1: nothing to gain from recomputing it
    assert oracle.strict_criterion(np.array([3.5], np.float32))[0] == 0.0


def brute_force_min_mask(kappa, tau):
    """Smallest q (fewest ones) with max_j (1 - q_j) kappa_j <= tau, by enumeration."""
    n = kappa.size
    for size in range(n + 1):
        sols = []
        for sel in itertools.combinations(range(n), size):
            q = np.zeros(n, dtype=bool)
            q[list(sel)] = True
            if np.all(np.where(q, 0.0, kappa) <= tau):
                sols.append(q)
        if sols:
            return sols
    raise AssertionError


@pytest.mark.parametrize("n", [3, 6, 9, 12])
def test_closed_form_equals_brute_force_minimum(n):
    rng = np.random.default_rng(n)
    for trial in range(6):
        y = (rng.standard_normal(n) * 1.5).astype(np.float32)
        kappa = jacobian_l1_columns_fd(y) * np.abs(y.astype(np.float64))
        ks = np.sort(kappa)
        # thresholds strictly between neighbouring kappa values (no ties)
        for t in range(n - 1):
            if ks[t + 1] - ks[t] < 1e-5 * max(ks[t + 1], 1e-12):
                continue
            tau = 0.5 * (ks[t] + ks[t + 1])
            sols = brute_force_min_mask(kappa, tau)
            assert len(sols) == 1, "the minimiser must be unique away from ties"
            closed = oracle.strict_criterion(y) > tau
            assert np.array_equal(closed, sols[0])


def test_s_rest_form_matches_plain_form_on_benign_rows():
    rng = np.random.default_rng(3)
    for _ in range(20):
        y = (rng.standard_normal(50)).astype(np.float32)
        z = softmax64(y)
        plain = 2 * z * (1 - z) * np.abs(y.astype(np.float64))
        assert np.allclose(oracle.strict_criterion(y), plain, rtol=1e-12, atol=1e-300)


def test_no_cancellation_near_z_equal_one():
    """A dominant maximum: 1 - z_a is tiny and must keep full relative accuracy."""
    y = np.array([40.0, 0.0, -1.0, 0.5], dtype=np.float32)
    c = oracle.strict_criterion(y)
    rest = np.exp(np.array([0.0, -1.0, 0.5]) - 40.0)
    one_minus_z = rest.sum() / (1 + rest.sum())
    z = 1 / (1 + rest.sum())
    assert c[0] == pytest.approx(2 * z * one_minus_z * 40.0, rel=1e-13)


def test_relaxed_bounds_strict_elementwise():
    """exp(y - M_running) >= exp(y - m) >= z and 1 - z <= 1, so every relaxed
    value bounds the strict one: relaxed selects a superset at equal tau."""
    rng = np.random.default_rng(4)
    for n in (5, 64, 65, 200, 1000):
        y = (rng.standard_normal(n) * 3).astype(np.float32)
        cs, cr = oracle.strict_criterion(y), oracle.relaxed_criterion(y)
        assert np.all(cr >= cs * (1 - 1e-15))


def test_relaxed_single_tile_identity():
    """Within one 64-key tile M is the row max, so c_relaxed = c_strict * S / (1 - z)."""
    rng = np.random.default_rng(5)
    y = (rng.standard_normal(64) * 2).astype(np.float32)
    yd = y.astype(np.float64)
    S = np.exp(yd - yd.max()).sum()
    z = softmax64(y)
    cs, cr = oracle.strict_criterion(y), oracle.relaxed_criterion(y)
    assert np.allclose(cr, cs * S / (1 - z), rtol=1e-12)


def test_relaxed_uses_the_running_max_of_64_key_tiles():
    y = np.zeros(192, dtype=np.float32)
    y[10] = 1.0      # tile 0 max
    y[100] = 5.0     # tile 1 raises the max
    y[150] = 3.0
    cr = oracle.relaxed_criterion(y)
    # tile 0 entries see M = 1 even though a larger score comes later
    assert cr[10] == pytest.approx(2.0 * 1.0, rel=1e-15)
    assert cr[100] == pytest.approx(2.0 * 5.0, rel=1e-15)
    assert cr[150] == pytest.approx(2 * math.exp(-2.0) * 3.0, rel=1e-14)
    assert cr[3] == 0.0  # |y| = 0


def test_selection_invariants_on_a_workload_slice():
    import synthetic as S
    w = S.Workload(1, 2, 96, 96, 64, seed=7)
    Q, K, V = S.make_qkv(w)
    counts = []
    for tau in (-1.0, 0.0, 0.01, 0.05, 0.2, np.inf):
        r = oracle.attention_rows(Q, K, V, mu=4, tau=tau)
        counts.append(int(r.nsel.sum()))
        if tau < 0:
            assert counts[-1] == w.valid_scores()            # everything recomputed
            assert np.array_equal(r.mixed.view(np.uint32), r.y32.view(np.uint32))
        if tau == np.inf:
            assert counts[-1] == 0
            assert np.array_equal(r.mixed.view(np.uint32), r.ps.view(np.uint32))
    assert counts == sorted(counts, reverse=True)             # monotone in tau
    # strict is a subset of relaxed at equal tau
    rs = oracle.attention_rows(Q, K, V, mu=4, tau=0.05, variant=oracle.STRICT)
    rr = oracle.attention_rows(Q, K, V, mu=4, tau=0.05, variant=oracle.RELAXED)
    assert np.all((rs.mask & ~rr.mask) == 0)


def test_tau_calibration_hits_the_requested_count():
    import synthetic as S
    w = S.Workload(1, 1, 128, 128, 64, seed=0)
    Q, K, V = S.make_qkv(w)
    r = oracle.attention_rows(Q, K, V, mu=4, tau=np.inf, want_crit=True)
    nv = [w.valid_keys(i) for i in range(128)]
    for rate in (0.003, 0.016, 0.076):
        tau = oracle.calibrate_tau(r.crit, nv, rate)
        r2 = oracle.attention_rows(Q, K, V, mu=4, tau=tau)
        k = round(rate * w.valid_scores())
        vals = np.concatenate([r.crit[i, :n] for i, n in enumerate(nv)])
        # PS scores are coarse, so criterion values tie; the count is the number
        # of values strictly above tau, which is at most k
        assert r2.nsel.sum() == np.sum(vals > tau)
        assert 0.9 * k <= r2.nsel.sum() <= k

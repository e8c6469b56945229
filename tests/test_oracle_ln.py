"""Pins of the LayerNorm oracle (LayerNorm after a PS(mu) linear map, greedy
recompute by sorted magnitude) to things other than itself: PyTorch's
layer_norm and its autograd Jacobian (whose 2-norm is the 1/sigma the bound
uses), the first-order bound on random perturbations, brute force over every
recompute set for minimality, and the special cases tau = +inf, tau < 0, mu = 23.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
import synthetic as S

EPS = oracle.LN_EPS


def torch_ln(y):
    t = torch.as_tensor(y, dtype=torch.float64)
    return torch.nn.functional.layer_norm(t, (t.shape[-1],), eps=EPS)


def test_layernorm_matches_torch():
    rng = np.random.default_rng(1)
    for n in (1, 2, 7, 64, 1600):
        y = rng.standard_normal(n) * rng.uniform(0.1, 10) + rng.uniform(-3, 3)
        out, sigma = oracle.layernorm(y)
        assert np.allclose(out, torch_ln(y).numpy(), rtol=1e-12, atol=1e-12)
        assert sigma == pytest.approx(np.sqrt(np.var(y) + EPS), rel=1e-14)


@pytest.mark.parametrize("n", [3, 8, 50])
def test_jacobian_two_norm_is_one_over_sigma(n):
    y = np.random.default_rng(n).standard_normal(n) * 2.0 + 0.5
    J = torch.autograd.functional.jacobian(lambda t: torch.nn.functional.layer_norm(t, (n,), eps=EPS),
                                           torch.tensor(y, dtype=torch.float64))
    _, sigma = oracle.layernorm(y)
    assert torch.linalg.matrix_norm(J, ord=2).item() == pytest.approx(1.0 / sigma, rel=1e-9)


def test_first_order_bound_holds_on_random_perturbations():
    rng = np.random.default_rng(2)
    y = rng.standard_normal(200).astype(np.float32)
    for tau in (2.0, 6.0, 12.0):
        sel, k, rest = oracle.ln_select(y, tau)
        _, sigma = oracle.layernorm(y.astype(np.float64))
        yd = y.astype(np.float64)
        base = torch_ln(yd).numpy()
        for _ in range(20):
            d = rng.uniform(-1e-6, 1e-6, size=y.size) * (1 - sel)
            moved = np.linalg.norm(torch_ln(yd * (1 + d)).numpy() - base)
            bound = np.sqrt(rest) / sigma * np.abs(d).max()
            assert moved <= bound * (1 + 1e-3)
        assert np.sqrt(rest) / sigma <= tau


def brute_force_min_count(y, tau):
    _, sigma = oracle.layernorm(y.astype(np.float64))
    best = None
    for q in itertools.product((0, 1), repeat=y.size):
        rest = sum(float(v) ** 2 for v, qj in zip(y, q) if not qj)
        if np.sqrt(rest) <= tau * sigma:
            c = sum(q)
            best = c if best is None else min(best, c)
    return best


@pytest.mark.parametrize("seed", range(5))
def test_greedy_is_a_sparsest_feasible_set(seed):
    rng = np.random.default_rng(100 + seed)
    y = (rng.standard_normal(10) * 1.5).astype(np.float32)
    t = oracle.ln_thresholds(y)
    # away from the threshold values themselves, where the two sides of the
    # comparison differ only by rounding
    for tau in (0.0, 0.5, 1.0, 2.0, 3.0, 0.5 * float(t[4] + t[5]), float(t[8]) * (1 + 1e-9), 100.0):
        sel, k, rest = oracle.ln_select(y, tau)
        assert k == brute_force_min_count(y, tau)
        # the set is the k largest magnitudes
        order = sorted(range(10), key=lambda j: (-abs(float(y[j])), j))
        assert set(np.nonzero(sel)[0]) == set(order[:k])
        # and the count changes where the thresholds say
        assert k == 10 - int(np.searchsorted(t, tau, side="right"))


def test_equal_magnitudes_go_in_ascending_index_order():
    y = np.array([1.0, -3.0, 3.0, 0.5, -3.0, 2.0], dtype=np.float32)
    t = oracle.ln_thresholds(y)
    tau = 0.5 * (t[3] + t[4])  # leaves the 4 smallest unselected: two of the three 3.0s selected
    sel, k, _ = oracle.ln_select(y, tau)
    assert k == 2 and list(np.nonzero(sel)[0]) == [1, 2]


def test_special_cases_and_layout():
    lw = S.LinearWorkload(24, 300, 64, seed=7)
    x, W = S.make_linear(lw)
    none = oracle.linear_ln_rows(x, W, scale=lw.scale, mu=4, tau=float("inf"))
    every = oracle.linear_ln_rows(x, W, scale=lw.scale, mu=4, tau=-1.0)
    f32 = oracle.linear_ln_rows(x, W, scale=lw.scale, mu=23, tau=float("inf"))
    assert none.nsel.sum() == 0 and every.nsel.sum() == lw.outputs()
    assert np.array_equal(every.mixed.view(np.uint32), f32.ps.view(np.uint32))
    assert np.allclose(every.out, f32.out, rtol=0, atol=0)
    assert np.allclose(none.out, torch_ln(none.ps.astype(np.float64)).numpy(), rtol=1e-12, atol=1e-12)
    # the linear map is the activation oracle's (pinned in test_oracle_act.py)
    g = oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=4, tau=float("inf"))
    assert np.array_equal(none.ps.view(np.uint32), g.ps.view(np.uint32))
    # counts never grow with tau
    counts = [oracle.linear_ln_rows(x, W, scale=lw.scale, mu=4, tau=t).nsel.sum() for t in (1, 5, 10, 15, 17)]
    assert all(a >= b for a, b in zip(counts, counts[1:]))


def test_error_falls_with_the_rate_and_greedy_beats_random():
    lw = S.LinearWorkload(48, 1600, 256, seed=8)
    x, W = S.make_linear(lw)
    full = oracle.linear_ln_rows(x, W, scale=lw.scale, mu=4, tau=-1.0, threads=4)
    base = oracle.linear_ln_rows(x, W, scale=lw.scale, mu=4, tau=float("inf"), threads=4)
    e_base = oracle.ln_errors(base.out, full.out)
    last = e_base["mean_l2"]
    for tau in (38.0, 36.0, 30.0):
        r = oracle.linear_ln_rows(x, W, scale=lw.scale, mu=4, tau=tau, threads=4)
        e = oracle.ln_errors(r.out, full.out)
        rnd = oracle.linear_ln_rows(x, W, scale=lw.scale, mu=4, variant=oracle.GIVEN_MASK,
                                    mask_in=S.linear_random_mask(lw, r.nsel), threads=4)
        e_rnd = oracle.ln_errors(rnd.out, full.out)
        assert e["mean_l2"] < last and e["mean_l2"] < e_rnd["mean_l2"]
        last = e["mean_l2"]


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=60, deadline=None)
@given(st.lists(st.floats(min_value=-6, max_value=6, allow_nan=False, width=32), min_size=2, max_size=9),
       st.floats(min_value=0.0, max_value=4.0))
def test_greedy_minimality_on_random_rows(vals, tau):
    """For any small row and tau: the greedy's count is the brute-force minimum,
    its set is feasible, and it is the top-k by magnitude (ties by index)."""
    y = np.array(vals, dtype=np.float32)
    t = oracle.ln_thresholds(y)
    if np.any(np.abs(t - tau) <= 1e-12 * max(1.0, tau)):
        return  # a threshold value itself: only rounding decides there
    sel, k, rest = oracle.ln_select(y, tau)
    assert k == brute_force_min_count(y, tau)
    order = sorted(range(y.size), key=lambda j: (-abs(float(y[j])), j))
    assert set(np.nonzero(sel)[0]) == set(order[:k])
    _, sigma = oracle.layernorm(y.astype(np.float64))
    if tau >= 0 and k < y.size:
        assert np.sqrt(rest) <= tau * sigma * (1 + 1e-12)

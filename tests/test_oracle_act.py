"""Pins of the activation oracle (GELU after a PS(mu) linear map) to things other
than itself: PyTorch's own tanh-form GELU, its autograd derivative and finite
differences for the condition number, brute force over every recompute set for
the selection, a plain float32 loop for the linear map's layout, and the special
cases of the method (tau = +inf, tau < 0, mu = 23).
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
import synthetic as S


def torch_gelu(y):
    return torch.nn.functional.gelu(torch.as_tensor(y, dtype=torch.float64), approximate="tanh")


def test_gelu_matches_torch_tanh_form():
    y = np.concatenate([np.linspace(-12, 12, 2001), [0.0, -0.75, 1e-8, -1e-8, 40.0, -40.0]])
    ref = torch_gelu(y).numpy()
    got = oracle.gelu(y)
    # 1 + tanh(u) cancels for very negative y: both sides are then within an
    # absolute |y| * 2^-52 of the true value
    assert np.all(np.abs(got - ref) <= 1e-14 * np.abs(ref) + 4e-16 * np.maximum(1.0, np.abs(y)))


def kappa_autograd(y):
    t = torch.tensor(y, dtype=torch.float64, requires_grad=True)
    f = torch_gelu(t)
    (g,) = torch.autograd.grad(f.sum(), t)
    return np.abs(y * g.numpy() / f.detach().numpy())


def test_kappa_matches_autograd_derivative():
    y = np.linspace(-6, 6, 1201)
    y = y[np.abs(y) > 1e-6]
    assert np.allclose(oracle.gelu_kappa(y), kappa_autograd(y), rtol=1e-11, atol=1e-12)


def test_kappa_matches_finite_differences():
    y = np.linspace(-5, 7, 241)
    y = y[np.abs(y) > 1e-3]
    h = 1e-5 * np.maximum(1.0, np.abs(y))
    fd = (torch_gelu(y + h).numpy() - torch_gelu(y - h).numpy()) / (2 * h)
    k_fd = np.abs(y * fd / torch_gelu(y).numpy())
    k = oracle.gelu_kappa(y)
    assert np.all(np.abs(k - k_fd) <= 1e-6 * np.maximum(1.0, k))


def test_kappa_in_high_precision_where_double_gelu_underflows():
    """60-digit decimal arithmetic: f(y) = y / (1 + e^(-2u)) has no cancellation,
    and a central difference with h = 1e-25 gives y f'(y) / f(y) to ~1e-40."""
    from decimal import Decimal, getcontext

    getcontext().prec = 60
    c = (Decimal(2) / Decimal("3.14159265358979323846264338327950288419716939937510582097494")).sqrt()
    a = Decimal("0.044715")

    def f(v):
        u = c * (v + a * v * v * v)
        return v / (1 + (-2 * u).exp())

    h = Decimal("1e-25")
    for yv in (-40.0, -25.0, -12.5, -8.0, -6.0, -3.3, -0.4, 0.6, 2.5, 9.0):
        v = Decimal(yv)
        kd = abs(v * (f(v + h) - f(v - h)) / (2 * h) / f(v))
        assert oracle.gelu_kappa(yv) == pytest.approx(float(kd), rel=2e-13)


def test_kappa_special_values():
    assert oracle.gelu_kappa(0.0) == 1.0           # the limit of y f'/f at 0
    assert abs(oracle.gelu_kappa(50.0) - 1.0) < 1e-15  # f(y) -> y
    # at GELU's minimum f' = 0: a perturbation of y leaves f unchanged to first order
    lo, hi = -1.0, -0.5
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        t = torch.tensor(mid, dtype=torch.float64, requires_grad=True)
        (g,) = torch.autograd.grad(torch_gelu(t), t)
        lo, hi = (mid, hi) if g.item() < 0 else (lo, mid)
    assert oracle.gelu_kappa(0.5 * (lo + hi)) < 1e-12
    # very negative inputs: f underflows to 0 but 1 - tanh u -> 2 and kappa stays finite
    c, a = np.sqrt(2 / np.pi), 0.044715
    for y in (-30.0, -200.0):
        assert oracle.gelu_kappa(y) == pytest.approx(abs(1 + 2 * y * c * (1 + 3 * a * y * y)), rel=1e-14)
    assert oracle.gelu_kappa(float("inf")) == float("inf")
    assert oracle.gelu_kappa(float("nan")) == float("inf")


def brute_force_min_set(kappa, tau):
    """Every q in {0,1}^n with max_j (1 - q_j) kappa_j <= tau; the ones of least
    cardinality."""
    n = len(kappa)
    best, sets = None, []
    for q in itertools.product((0, 1), repeat=n):
        worst = max([k for k, qj in zip(kappa, q) if not qj], default=0.0)
        if worst <= tau:
            c = sum(q)
            if best is None or c < best:
                best, sets = c, [q]
            elif c == best:
                sets.append(q)
    return sets


@pytest.mark.parametrize("seed", range(6))
def test_selection_is_the_unique_sparsest_feasible_set(seed):
    lw = S.LinearWorkload(1, 10, 16, seed=seed)
    x, W = S.make_linear(lw)
    r = oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=3, tau=0.0, variant=oracle.STRICT)
    kappa = r.kappa[0]
    for tau in (0.0, 0.5, 1.0, 1.2, 2.0, float(np.median(kappa)), float(kappa.max())):
        r = oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=3, tau=tau, variant=oracle.STRICT)
        sets = brute_force_min_set(list(kappa), tau)
        assert len(sets) == 1
        bits = [(int(r.mask[0, 0]) >> j) & 1 for j in range(10)]
        assert tuple(bits) == sets[0]
        assert r.nsel[0] == sum(bits)


def test_linear_map_layout_against_a_float32_loop():
    lw = S.LinearWorkload(3, 5, 8, seed=3)
    x, W = S.make_linear(lw)
    xf, wf = S.bf16_bits_to_f32(x), S.bf16_bits_to_f32(W)
    scale = np.float32(lw.scale)
    r = oracle.linear_gelu_rows(x, W, scale=scale, mu=23, tau=float("inf"))
    for i in range(3):
        for j in range(5):
            acc = np.float32(0.0)
            for k in range(8):
                acc = np.float32(acc + np.float32(xf[i, k] * wf[j, k]))
            assert r.ps[i, j] == np.float32(scale * acc)
    # PS(4): every output is the pinned PS(mu) dot product of row i of x and row j of W
    r4 = oracle.linear_gelu_rows(x, W, scale=scale, mu=4, tau=float("inf"))
    for i in range(3):
        for j in range(5):
            assert r4.ps[i, j] == oracle.ps_dot(x[i], W[j], 4, float(scale))


def test_special_cases():
    lw = S.LINEAR_WORKLOADS["gelu_small_96x300x200"]
    x, W = S.make_linear(lw)
    rows = np.arange(0, lw.M, 7)
    none = oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=4, tau=float("inf"), rows=rows)
    every = oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=4, tau=-1.0, rows=rows)
    f32 = oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=23, tau=float("inf"), rows=rows)
    assert none.nsel.sum() == 0 and np.array_equal(none.mixed, none.ps)
    assert every.nsel.sum() == rows.size * lw.N
    assert np.array_equal(every.mixed.view(np.uint32), f32.ps.view(np.uint32))  # FP32 recompute = PS(23)
    assert np.array_equal(every.out, f32.out)
    assert np.array_equal(none.out, oracle.gelu(none.ps))
    # tau = 0 selects every output with kappa > 0 (all of them for these inputs)
    zero = oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=4, tau=0.0, rows=rows)
    assert zero.nsel.sum() == int((zero.kappa > 0).sum())
    # the count never grows with tau
    counts = [oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=4, tau=t, rows=rows).nsel.sum()
              for t in (0.5, 1.0, 1.3, 2.0, 4.0, 10.0)]
    assert all(a >= b for a, b in zip(counts, counts[1:]))


def test_amplification_falls_with_the_rate_and_adaptive_beats_random():
    """The kappa test bounds how much an output amplifies its input's relative
    error; a random choice of the same per-row count does not."""
    lw = S.LINEAR_WORKLOADS["gelu_small_96x300x200"]
    x, W = S.make_linear(lw)
    full = oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=4, tau=-1.0, threads=4)
    base = oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=4, tau=float("inf"), threads=4)
    e_base = oracle.act_errors(base.out, base.mixed, full.out, full.mixed)
    errs = []
    for rate in (0.003, 0.016, 0.076):
        tau = oracle.calibrate_tau(base.kappa, [lw.N] * lw.M, rate)
        r = oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=4, tau=tau, threads=4)
        errs.append(oracle.act_errors(r.out, r.mixed, full.out, full.mixed))
        if rate == 0.016:
            mask = S.linear_random_mask(lw, r.nsel)
            rnd = oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=4, variant=oracle.GIVEN_MASK,
                                          mask_in=mask, threads=4)
            assert rnd.nsel.sum() == r.nsel.sum()
            e_rnd = oracle.act_errors(rnd.out, rnd.mixed, full.out, full.mixed)
            assert errs[-1]["max_amp"] < 0.5 * e_rnd["max_amp"]
            assert e_rnd["max_amp"] > 0.5 * e_base["max_amp"]
    assert errs[0]["max_amp"] < e_base["max_amp"]
    assert errs[0]["max_amp"] > errs[1]["max_amp"] > errs[2]["max_amp"]
    # recomputed components carry no error, and the selections are nested
    assert e_base["l1_rel"] > errs[0]["l1_rel"] > errs[1]["l1_rel"] > errs[2]["l1_rel"]


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=200, deadline=None)
@given(st.floats(min_value=-8, max_value=8, allow_nan=False))
def test_kappa_matches_autograd_on_random_inputs(y):
    if abs(y) < 1e-6:
        return
    k = oracle.gelu_kappa(y)
    ref = kappa_autograd(np.array([y]))[0]
    f = float(torch_gelu(np.array([y]))[0])
    if abs(f) < 1e-12:  # double GELU underflows in PyTorch's form; the decimal pin covers it
        return
    assert k == pytest.approx(ref, rel=1e-9, abs=1e-10)

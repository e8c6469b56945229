"""PS(mu) and binary32 key-query scores of the oracle, pinned outside the oracle.

LAMP summary, "Implementation strategy" step 1 (low-precision baseline of g)
and step 3 (recompute in FP32); "Experimental results" (PS(mu)).
"""
import os

import numpy as np
import pytest

import oracle
from tests.test_oracle_round import grid_nearest
import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ps_dot.txt")


def bf16(vals):
    return S.to_bf16_bits(np.asarray(vals, dtype=np.float64))


def test_golden_hand_cases():
    n = 0
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if not line:
            continue
        mu, scale, qs, ks, want_ps, want_32 = [f.strip() for f in line.split("|")]
        q = bf16([float(v) for v in qs.split()])
        k = bf16([float(v) for v in ks.split()])
        assert np.array_equal(S.bf16_bits_to_f32(q), np.array([float(v) for v in qs.split()], np.float32))
        got = oracle.ps_dot(q, k, int(mu), float(scale))
        got32 = oracle.fp32_dot(q, k, float(scale))
        assert got == np.float32(float(want_ps)), (line, got)
        assert got32 == np.float32(float(want_32)), (line, got32)
        n += 1
    assert n >= 8


def sequential_ps_reference(q_bits, k_bits, mu, scale):
    """The PS(mu) sum composed from numpy float32 arithmetic and the independent
    grid-nearest rounding of the rounding tests."""
    qf = S.bf16_bits_to_f32(q_bits)
    kf = S.bf16_bits_to_f32(k_bits)
    acc = np.float32(0.0)
    for t in range(qf.size):
        acc = grid_nearest(np.array([np.float32(acc + np.float32(qf[t] * kf[t]))]), mu)[0]
    return np.float32(np.float32(scale) * acc)


@pytest.mark.parametrize("mu", [1, 3, 4, 6, 7, 10, 15, 22])
def test_ps_dot_against_composed_reference(mu):
    w = S.Workload(1, 1, 16, 16, 64, causal=False, seed=11)
    Q, K, _ = S.make_qkv(w)
    sc = oracle.default_scale(64)
    for i in range(16):
        for j in range(0, 16, 3):
            assert oracle.ps_dot(Q[0, 0, i], K[0, 0, j], mu, sc) == \
                sequential_ps_reference(Q[0, 0, i], K[0, 0, j], mu, sc)


def test_mu23_scores_equal_binary32_scores():
    w = S.Workload(1, 2, 64, 64, 128, causal=False, seed=2)
    Q, K, V = S.make_qkv(w)
    r = oracle.attention_rows(Q, K, V, causal=False, mu=23, tau=np.inf)
    assert np.array_equal(r.ps.view(np.uint32), r.y32.view(np.uint32))


def test_fp32_scores_are_sequential_binary32_sums():
    """numpy's add.accumulate runs strictly left to right in float32: an
    independent sequential binary32 sum (bf16 products are exact in binary32)."""
    w = S.Workload(1, 1, 32, 48, 128, causal=False, seed=3)
    Q, K, V = S.make_qkv(w)
    r = oracle.attention_rows(Q, K, V, causal=False, mu=4, tau=np.inf)
    qf = S.bf16_bits_to_f32(Q[0, 0])
    kf = S.bf16_bits_to_f32(K[0, 0])
    sc = np.float32(oracle.default_scale(128))
    for i in range(32):
        prods = (qf[i][None, :] * kf).astype(np.float32)
        seq = np.add.accumulate(prods, axis=1, dtype=np.float32)[:, -1]
        assert np.array_equal((sc * seq).astype(np.float32).view(np.uint32), r.y32[i].view(np.uint32))


def test_fp32_scores_within_higham_bound_of_exact():
    w = S.Workload(1, 1, 8, 256, 64, causal=False, seed=4)
    Q, K, V = S.make_qkv(w)
    r = oracle.attention_rows(Q, K, V, causal=False, mu=4, tau=np.inf)
    qf = S.bf16_bits_to_f32(Q[0, 0]).astype(np.float64)
    kf = S.bf16_bits_to_f32(K[0, 0]).astype(np.float64)
    sc = oracle.default_scale(64)
    exact = sc * (qf @ kf.T)
    absum = sc * (np.abs(qf) @ np.abs(kf).T)
    u = 2.0 ** -24
    gamma = 64 * u / (1 - 64 * u)
    assert np.all(np.abs(r.y32 - exact) <= gamma * absum + 1e-30)
    # and the PS(4) scores differ from exact by at most the mu-bit analogue
    u4 = 2.0 ** -5
    g4 = ((1 + u4) * (1 + u)) ** 64 - 1
    assert np.all(np.abs(r.ps - exact) <= g4 * absum)
    # PS(4) is visibly coarser than binary32 on average
    assert np.mean(np.abs(r.ps - exact)) > 100 * np.mean(np.abs(r.y32 - exact))

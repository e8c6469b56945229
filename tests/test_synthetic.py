"""Seeded synthetic inputs shared by the CUDA path's tests and the oracle's."""
import numpy as np

import synthetic as S


def test_splitmix64_reference_values():
    # SplitMix64 seeded with 0: the first outputs of the published generator
    first = S.mix64(np.array([0x9E3779B97F4A7C15, 2 * 0x9E3779B97F4A7C15 % 2**64], dtype=np.uint64))
    assert [int(v) for v in first] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4]


def test_deterministic_and_counter_based():
    w = S.Workload(1, 2, 8, 8, 64, seed=5)
    a = S.make_tensor(w, S.STREAM_Q, 8)
    b = S.make_tensor(w, S.STREAM_Q, 8)
    assert np.array_equal(a, b)
    # element n depends only on (seed, stream, n)
    part = S.normal_f64(5, S.STREAM_Q, 100, 10)
    full = S.normal_f64(5, S.STREAM_Q, 0, 110)
    assert np.array_equal(part, full[100:])
    assert not np.array_equal(S.make_tensor(w, S.STREAM_K, 8), a)


def test_normal_moments_and_bf16_exactness():
    x = S.normal_f64(0, 0, 0, 400000)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    bits = S.to_bf16_bits(x[:1000])
    f = S.bf16_bits_to_f32(bits)
    assert np.all(np.abs(f - x[:1000]) <= np.abs(x[:1000]) * 2.0 ** -8 + 1e-30)


def test_outlier_channels_scaled_in_q_and_k_only():
    w = S.Workload(1, 3, 64, 64, 64, outlier_frac=0.01, seed=0)
    ch = S.outlier_channels(w)
    assert ch.shape == (3, 1)
    Q, K, V = (S.bf16_bits_to_f32(t) for t in S.make_qkv(w))
    for bh in range(3):
        c = ch[bh, 0]
        for T in (Q, K):
            assert np.abs(T[0, bh][:, c]).mean() > 10 * np.abs(np.delete(T[0, bh], c, axis=1)).mean()
        assert np.abs(V[0, bh][:, c]).mean() < 2


def test_random_control_mask_counts_and_validity():
    w = S.Workload(1, 2, 50, 60, 64, seed=1)
    rng = np.random.default_rng(0)
    nv = np.array([w.valid_keys(i) for i in range(50)])
    counts = np.stack([rng.integers(0, nv + 1) for _ in range(2)])
    m = S.random_control_mask(w, counts)
    bits = S.unpack_mask(m, 60)
    assert np.array_equal(bits.sum(-1), counts)
    for i in range(50):
        assert not bits[:, i, nv[i]:].any()
    assert np.array_equal(S.pack_mask(bits), m)


def test_linear_workload_inputs():
    lw = S.LinearWorkload(5, 40, 24, seed=2)
    x, W = S.make_linear(lw)
    x2, W2 = S.make_linear(lw)
    assert x.shape == (5, 24) and W.shape == (40, 24) and x.dtype == np.uint16
    assert np.array_equal(x, x2) and np.array_equal(W, W2)
    assert not np.array_equal(x[0, :24], W[0, :24])          # x and W use separate streams
    assert lw.scale == np.float32(1 / np.sqrt(24))
    xf = S.bf16_bits_to_f32(S.make_linear(S.LinearWorkload(64, 64, 256, seed=1))[0])
    assert abs(float(xf.mean())) < 0.02 and abs(float(xf.std()) - 1) < 0.02


def test_linear_random_mask_counts():
    lw = S.LinearWorkload(7, 70, 8, seed=4)
    counts = np.array([0, 1, 5, 70, 3, 33, 2])
    m = S.linear_random_mask(lw, counts)
    bits = S.unpack_mask(m, lw.N)
    assert m.shape == (7, 3) and np.array_equal(bits.sum(axis=1), counts)
    assert int(m[:, -1].max()) >> 6 == 0                     # no bits past N

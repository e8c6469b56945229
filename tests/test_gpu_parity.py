"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Small problems are compared on every row; the full-size workloads on sampled
rows (the oracle computes each row on its own) plus properties that hold at any
size. Bars: see tests/parity.py.
"""
import numpy as np
import pytest
import torch

import mixed_precision_attention_ps_b200 as lamp
import oracle
import synthetic as S
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lamp.load()


def run_case(w, mu, tau, variant, rows=None, mask_in=None, scale=0.0, threads=8):
    Q, K, V = S.make_qkv(w)
    g = P.GpuCall(w, P.to_device(Q), P.to_device(K), P.to_device(V), mu=mu, tau=tau, variant=variant,
                 mask_in=None if mask_in is None else torch.from_numpy(mask_in.view(np.int32)).cuda(),
                 scale=scale)
    if rows is None:
        rows = np.arange(w.B * w.H * w.n_q, dtype=np.int64)
    orc = oracle.attention_rows(Q, K, V, causal=w.causal, scale=scale or None, mu=mu, tau=tau,
                                variant=variant, mask_in=mask_in, rows=rows, want_crit=True,
                                threads=threads)
    stats = P.compare(w, g.rows(rows), orc, rows, tau, variant)
    return g, orc, stats


# --------------------------------------------------------------------------------------
# every row of small problems
# --------------------------------------------------------------------------------------

def test_single_head_128_strict_mu4():
    """The small workload: 1 head, causal 128 x 128, d = 64, strict, mu = 4, tau = 0.05."""
    w = S.WORKLOADS["single_head_128"]
    g, orc, st = run_case(w, 4, 0.05, oracle.STRICT)
    assert g.count() == int(orc.nsel.sum()) > 0
    print(st)


@pytest.mark.parametrize("B,H,n_q,n_k,d,causal", [
    (1, 1, 1, 1, 64, True),        # one query, one key
    (1, 2, 37, 37, 64, True),      # ragged: below one tile
    (2, 3, 100, 100, 64, True),    # several row blocks, ragged tail
    (1, 1, 200, 333, 64, True),    # n_k > n_q: bottom-right causal alignment
    (1, 1, 150, 90, 64, True),     # n_q > n_k: the first 60 rows see no key
    (1, 2, 70, 257, 64, False),    # non-causal, n_k one past a tile boundary
    (1, 1, 64, 64, 128, True),     # d = 128
    (1, 2, 161, 129, 128, False),  # d = 128, ragged
    (1, 1, 40, 1500, 64, False),   # streamed: three 512-key tiles, the last one ragged
    (1, 1, 33, 1100, 128, True),   # d = 128 streamed, just past the whole-row limit
    (1, 1, 20, 3000, 64, False),   # streamed: six tiles
    (1, 2, 19, 3000, 128, True),   # d = 128 streamed, causal with n_k > n_q
    (1, 1, 24, 5000, 64, False),   # streamed: ten tiles
    (1, 1, 9, 4700, 128, True),    # d = 128 streamed, nine tiles plus a ragged one
])
@pytest.mark.parametrize("variant", [oracle.STRICT, oracle.RELAXED])
def test_shapes(B, H, n_q, n_k, d, causal, variant):
    w = S.Workload(B, H, n_q, n_k, d, causal=causal, seed=B * 1000 + n_q + n_k + d)
    run_case(w, 4, 0.02, variant)


@pytest.mark.parametrize("mu", [1, 2, 3, 6, 7, 10, 11, 13, 16, 22, 23])
def test_every_rounding_class(mu):
    w = S.Workload(1, 2, 96, 96, 64, seed=mu)
    run_case(w, mu, 0.01, oracle.STRICT)


@pytest.mark.parametrize("tau", [-1.0, 0.0, 1e-3, 0.3, float("inf")])
@pytest.mark.parametrize("variant", [oracle.STRICT, oracle.RELAXED])
def test_threshold_special_cases(tau, variant):
    w = S.Workload(1, 2, 130, 130, 64, seed=3)
    g, orc, _ = run_case(w, 4, tau, variant)
    nsel = g.count()
    if tau < 0:
        assert nsel == w.valid_scores()
    if tau == float("inf"):
        assert nsel == 0


def test_tau_below_zero_and_mu23_are_fp32_attention():
    w = S.Workload(1, 2, 100, 100, 64, seed=4)
    Q, K, V = S.make_qkv(w)
    Qd, Kd, Vd = P.to_device(Q), P.to_device(K), P.to_device(V)
    a = P.GpuCall(w, Qd, Kd, Vd, mu=4, tau=-1.0, variant=oracle.STRICT)
    b = P.GpuCall(w, Qd, Kd, Vd, mu=23, tau=float("inf"), variant=oracle.STRICT)
    rows = np.arange(w.B * w.H * w.n_q)
    ra, rb = a.rows(rows), b.rows(rows)
    assert np.array_equal(ra["mixed"].view(np.uint32), rb["mixed"].view(np.uint32))
    assert np.array_equal(rb["ps"].view(np.uint32), rb["mixed"].view(np.uint32))
    assert np.array_equal(ra["out"], rb["out"])


def test_given_mask_random_control():
    w = S.Workload(2, 2, 120, 120, 64, seed=5)
    rng = np.random.default_rng(0)
    nv = np.array([w.valid_keys(i) for i in range(w.n_q)])
    counts = np.stack([rng.integers(0, nv // 4 + 1) for _ in range(w.B * w.H)])
    mask = S.random_control_mask(w, counts).reshape(w.B, w.H, w.n_q, -1)
    # junk bits on invalid keys and on the padding past n_k are ignored by both sides
    bits = S.unpack_mask(mask, w.n_k)
    invalid = np.arange(w.n_k)[None, :] >= nv[:, None]
    bits |= invalid[None, None] & (rng.random(bits.shape) < 0.5)
    mask = S.pack_mask(bits)
    mask[..., -1] |= np.uint32(0xFF000000)
    g, orc, _ = run_case(w, 4, 0.0, oracle.GIVEN_MASK, mask_in=mask)
    assert g.count() == int(counts.sum())


def test_explicit_scale():
    w = S.Workload(1, 1, 64, 80, 128, seed=6)
    run_case(w, 5, 0.05, oracle.STRICT, scale=0.3)


def test_outlier_channels():
    w = S.Workload(1, 2, 128, 128, 64, outlier_frac=0.01, seed=7)
    run_case(w, 4, 0.05, oracle.STRICT)
    run_case(w, 6, 0.05, oracle.RELAXED)


def test_nonfinite_free_extreme_inputs_take_the_exact_path():
    """Heads whose magnitudes could leave the fast rounding domain (very large or
    subnormal-range products) must still be bit-exact."""
    w = S.Workload(1, 3, 64, 64, 64, causal=False, seed=8)
    Q, K, V = S.make_qkv(w)
    Qf, Kf = S.bf16_bits_to_f32(Q).copy(), S.bf16_bits_to_f32(K).copy()
    Qf[0, 0] *= 2.0 ** 50     # huge products in head 0
    Kf[0, 0] *= 2.0 ** 50
    Qf[0, 1] *= 2.0 ** -70    # products below the normal range in head 1
    Kf[0, 1] *= 2.0 ** -70
    Q2 = S.to_bf16_bits(Qf.astype(np.float64)).reshape(Q.shape)
    K2 = S.to_bf16_bits(Kf.astype(np.float64)).reshape(K.shape)
    for mu in (4, 10, 23):
        g = P.GpuCall(w, P.to_device(Q2), P.to_device(K2), P.to_device(V), mu=mu, tau=0.05,
                     variant=oracle.STRICT, scale=1.0)
        rows = np.arange(w.B * w.H * w.n_q)
        orc = oracle.attention_rows(Q2, K2, V, causal=False, scale=1.0, mu=mu, tau=0.05, rows=rows,
                                    want_crit=True, threads=8)
        gr = g.rows(rows)
        assert np.array_equal(gr["ps"].view(np.uint32), orc.ps.view(np.uint32))


def test_repeated_calls_are_deterministic():
    w = S.Workload(1, 4, 256, 256, 64, seed=9)
    Q, K, V = S.make_qkv(w)
    Qd, Kd, Vd = P.to_device(Q), P.to_device(K), P.to_device(V)
    outs = [lamp.attention(Qd, Kd, Vd, mu=4, tau=0.02, want_count=True) for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.out, outs[0].out) and torch.equal(o.mask, outs[0].mask)
        assert o.n_selected.item() == outs[0].n_selected.item()


def test_caller_workspace_and_stream():
    w = S.Workload(1, 2, 100, 100, 64, seed=10)
    Q, K, V = S.make_qkv(w)
    Qd, Kd, Vd = P.to_device(Q), P.to_device(K), P.to_device(V)
    dims = (w.B, w.H, w.n_q, w.n_k, w.d)
    need = lamp.lamp_workspace_size(dims, lamp.LAMP_STRICT)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    out = torch.empty_like(Qd)
    mask = torch.zeros((1, 2, 100, 4), dtype=torch.int32, device="cuda")
    with pytest.raises(lamp.LampError) as ei:
        lamp.lamp_attention_ex(dims=dims, Q=Qd, K=Kd, V=Vd, out=out, mu=4, tau=0.03, stream=s,
                               workspace=ws, workspace_bytes=need - 1)
    assert ei.value.code == lamp.LAMP_ERR_WORKSPACE
    lamp.lamp_attention_ex(dims=dims, Q=Qd, K=Kd, V=Vd, out=out, mask_out=mask, mu=4, tau=0.03, stream=s,
                           workspace=ws, workspace_bytes=need)
    s.synchronize()
    ref = lamp.attention(Qd, Kd, Vd, mu=4, tau=0.03)
    torch.cuda.synchronize()
    assert torch.equal(out, ref.out) and torch.equal(mask, ref.mask)


# --------------------------------------------------------------------------------------
# device PS(mu) rounding utility
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("mu", [1, 4, 7, 10, 13, 22, 23])
def test_device_rounding_exact_path(mu):
    from tests.test_oracle_round import structured_sample
    x = structured_sample(mu, seed=mu)
    xd = torch.from_numpy(x.copy()).cuda()
    yd = torch.empty_like(xd)
    lamp.lamp_ps_round(xd, yd, x.size, mu, 0)
    torch.cuda.synchronize()
    want = oracle.round_ps(x, mu)
    assert np.array_equal(yd.cpu().numpy().view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("mu", [1, 2, 4, 6, 7, 9, 10])
def test_device_rounding_fast_path_in_its_domain(mu):
    """The two-instruction rounding equals the exact rounding for +0 and normal
    |x| < 2^(127 - (23 - mu)): all binary32 patterns of four binades around 1
    and every exponent with structured fractions."""
    from tests.test_oracle_round import structured_sample
    s = 23 - mu
    x = structured_sample(mu, seed=100 + mu)
    bits = x.view(np.uint32)
    e = ((bits >> 23) & 0xFF).astype(np.int64)
    dom = ((e >= 1) & (e - 127 < 127 - s)) | ((bits & 0x7FFFFFFF) == 0)
    dom &= bits != 0x80000000  # -0 never occurs as a partial sum
    dense = np.arange(0x3E800000, 0x40800000, dtype=np.uint32)  # [0.25, 4)
    x = np.concatenate([x[dom], dense.view(np.float32), -dense.view(np.float32)])
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    lamp.lamp_ps_round(xd, yd, x.size, mu, 1)
    torch.cuda.synchronize()
    want = oracle.round_ps(x, mu)
    assert np.array_equal(yd.cpu().numpy().view(np.uint32), want.view(np.uint32))


# --------------------------------------------------------------------------------------
# full-size workloads, sampled rows
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("mu,tau", [(4, 0.05), (7, 0.02), (10, 0.005)])
def test_gpt2xl_shape_strict_sampled(mu, tau):
    w = S.WORKLOADS["gpt2xl_1x25x1024x64"]
    rows = P.sample_rows(w, 24, 6, seed=mu)
    g, orc, st = run_case(w, mu, tau, oracle.STRICT, rows=rows)
    print(st)


def test_gpt2xl_shape_count_matches_mask_and_is_monotone():
    w = S.WORKLOADS["gpt2xl_1x25x1024x64"]
    Q, K, V = S.make_qkv(w)
    Qd, Kd, Vd = P.to_device(Q), P.to_device(K), P.to_device(V)
    prev = None
    for tau in (0.001, 0.01, 0.05, 0.2):
        r = lamp.attention(Qd, Kd, Vd, mu=4, tau=tau, want_count=True)
        torch.cuda.synchronize()
        m = r.mask.view(torch.int32).cpu().numpy().view(np.uint32)
        bits = int(np.unpackbits(m.view(np.uint8)).sum())
        assert bits == r.n_selected.item()
        if prev is not None:
            assert bits <= prev
        prev = bits


def test_batch8_relaxed_sampled():
    w = S.WORKLOADS["batch8_8x25x1024x64"]
    rows = P.sample_rows(w, 12, 8, seed=3)
    run_case(w, 4, 0.3, oracle.RELAXED, rows=rows)


def test_outlier_4x25x4096_strict_sampled():
    w = S.WORKLOADS["outlier_4x25x4096x64"]
    rows = P.sample_rows(w, 6, 5, seed=5)
    for mu, tau in ((4, 0.02), (6, 0.005)):
        run_case(w, mu, tau, oracle.STRICT, rows=rows)


def test_long_context_relaxed_sampled():
    w = S.WORKLOADS["long_1x32x16384x128"]
    rows = P.sample_rows(w, 3, 4, seed=7)
    run_case(w, 4, 0.5, oracle.RELAXED, rows=rows)

"""GPU parity of the decode path: a few query rows per head (n_q <= 4) against rows
of 512 keys or more, split over 512-key chunks (scores with chunk statistics,
selection with the row statistics combined across chunks, chunk softmax and
partial P.V, then the combine).

Compared with the CPU oracle through the C ABI, as in tests/test_gpu_parity.py:
low-precision and mixed scores and mask words bit-exact, outputs within the
parity bars. Shapes put row ends and n_k on, one past and one short of the chunk
and 64-key tile boundaries; the causal rows end at different keys.
"""
import numpy as np
import pytest
import torch

import mixed_precision_attention_ps_b200 as lamp
import oracle
import synthetic as S
from tests import parity as P
from tests.test_gpu_parity import run_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lamp.load()


@pytest.mark.parametrize("B,H,n_q,n_k,d,causal", [
    (1, 3, 1, 512, 64, True),       # one chunk exactly
    (1, 2, 1, 513, 128, True),      # a one-key second chunk
    (2, 2, 2, 1000, 64, True),      # causal rows ending one key apart
    (1, 4, 3, 1535, 128, False),    # one short of three chunks
    (1, 2, 4, 4099, 64, True),      # four rows, nine chunks
    (1, 1, 1, 16384, 128, True),    # a 16K-key cache
])
@pytest.mark.parametrize("variant", [oracle.STRICT, oracle.RELAXED])
def test_decode_shapes(B, H, n_q, n_k, d, causal, variant):
    w = S.Workload(B, H, n_q, n_k, d, causal=causal, seed=9000 + n_q + n_k + d)
    tau = 0.02 if variant == oracle.STRICT else 0.3
    g, orc, _ = run_case(w, 4, tau, variant)
    assert g.count() == int(orc.nsel.sum())


@pytest.mark.parametrize("mu", [1, 7, 10, 11, 16, 23])
def test_decode_rounding_classes(mu):
    w = S.Workload(1, 2, 2, 1200, 64, causal=False, seed=400 + mu)
    run_case(w, mu, 0.02, oracle.STRICT)


@pytest.mark.parametrize("tau", [-1.0, 0.0, 0.05, float("inf")])
@pytest.mark.parametrize("variant", [oracle.STRICT, oracle.RELAXED])
def test_decode_threshold_special_cases(tau, variant):
    w = S.Workload(1, 2, 1, 1100, 64, seed=41)
    g, orc, _ = run_case(w, 4, tau, variant)
    if tau < 0:
        assert g.count() == w.valid_scores()
    if tau == float("inf"):
        assert g.count() == 0


def test_decode_given_mask_with_junk_bits():
    w = S.Workload(1, 3, 2, 2100, 128, seed=42)
    rng = np.random.default_rng(42)
    nv = np.array([w.valid_keys(i) for i in range(w.n_q)])
    counts = np.stack([rng.integers(0, nv // 8 + 1) for _ in range(w.B * w.H)])
    mask = S.random_control_mask(w, counts).reshape(w.B, w.H, w.n_q, -1)
    bits = S.unpack_mask(mask, w.n_k)
    invalid = np.arange(w.n_k)[None, :] >= nv[:, None]
    bits |= invalid[None, None] & (rng.random(bits.shape) < 0.5)
    mask = S.pack_mask(bits)
    mask[..., -1] |= np.uint32(0xFFF00000)  # padding past n_k
    g, _, _ = run_case(w, 4, 0.0, oracle.GIVEN_MASK, mask_in=mask)
    assert g.count() == int(counts.sum())


def test_decode_outlier_channels_strict():
    w = S.Workload(1, 4, 1, 3000, 64, outlier_frac=0.01, seed=43)
    run_case(w, 4, 0.01, oracle.STRICT)


def test_decode_tau_below_zero_and_mu23_agree():
    """Every score recomputed (tau < 0) and PS(23) scores give the same binary32
    scores, and the same outputs."""
    w = S.Workload(1, 2, 2, 1800, 64, causal=False, seed=44)
    Q, K, V = S.make_qkv(w)
    Qd, Kd, Vd = P.to_device(Q), P.to_device(K), P.to_device(V)
    a = P.GpuCall(w, Qd, Kd, Vd, mu=4, tau=-1.0, variant=oracle.STRICT)
    b = P.GpuCall(w, Qd, Kd, Vd, mu=23, tau=float("inf"), variant=oracle.STRICT)
    rows = np.arange(w.B * w.H * w.n_q)
    ra, rb = a.rows(rows), b.rows(rows)
    assert np.array_equal(ra["mixed"].view(np.uint32), rb["mixed"].view(np.uint32))
    assert np.array_equal(ra["out"], rb["out"])


def test_decode_repeated_calls_are_deterministic():
    w = S.Workload(2, 4, 1, 5000, 128, seed=45)
    Q, K, V = S.make_qkv(w)
    Qd, Kd, Vd = P.to_device(Q), P.to_device(K), P.to_device(V)
    outs = [lamp.attention(Qd, Kd, Vd, mu=4, tau=0.02, want_count=True) for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.out, outs[0].out) and torch.equal(o.mask, outs[0].mask)
        assert o.n_selected.item() == outs[0].n_selected.item()

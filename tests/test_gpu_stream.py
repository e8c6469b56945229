"""GPU parity of the streamed one-pass path: the relaxed and given-mask variants
on rows too long for two whole 16-row score buffers in shared memory (more than
1024 keys), where scores go through 512-key tiles with an online softmax.

Compared with the CPU oracle through the C ABI, like tests/test_gpu_parity.py:
low-precision and mixed scores and mask words bit-exact, outputs within the
parity bars. The shapes put row ends, causal diagonals and n_k on, one past and
one short of the 512-key tile and 64-key sub-tile boundaries.
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
    (1, 1, 17, 1025, 64, False),    # one key past the whole-row limit; ragged 16-row item
    (1, 2, 33, 1536, 64, True),     # three full tiles, causal with n_k > n_q
    (1, 1, 20, 1537, 128, False),   # a one-key last tile
    (2, 1, 48, 2047, 64, True),     # one short of four tiles
    (1, 1, 600, 1100, 64, True),    # causal rows ending inside every tile
    (1, 1, 1300, 1200, 128, True),  # n_q > n_k: the first 100 rows see no key
    (1, 3, 9, 3000, 128, False),    # several heads, d = 128
])
def test_stream_shapes_relaxed(B, H, n_q, n_k, d, causal):
    w = S.Workload(B, H, n_q, n_k, d, causal=causal, seed=7000 + n_q + n_k + d)
    g, orc, _ = run_case(w, 4, 0.3, oracle.RELAXED)
    assert g.count() == int(orc.nsel.sum())


@pytest.mark.parametrize("mu", [1, 7, 10, 11, 16, 23])
def test_stream_rounding_classes(mu):
    w = S.Workload(1, 2, 24, 1300, 64, causal=False, seed=300 + mu)
    run_case(w, mu, 0.1, oracle.RELAXED)


@pytest.mark.parametrize("tau", [-1.0, 0.0, 0.05, float("inf")])
def test_stream_threshold_special_cases(tau):
    w = S.Workload(1, 1, 40, 1400, 64, seed=11)
    g, orc, _ = run_case(w, 4, tau, oracle.RELAXED)
    if tau < 0:
        assert g.count() == w.valid_scores()
    if tau == float("inf"):
        assert g.count() == 0


def test_stream_given_mask_with_junk_bits():
    w = S.Workload(1, 2, 40, 2100, 64, seed=12)
    rng = np.random.default_rng(12)
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


def test_stream_tau_below_zero_and_mu23_agree():
    """Every score recomputed (tau < 0) and PS(23) scores with nothing recomputed
    give the same binary32 scores, so the same outputs bit for bit."""
    w = S.Workload(1, 2, 30, 1800, 64, causal=False, seed=13)
    Q, K, V = S.make_qkv(w)
    Qd, Kd, Vd = P.to_device(Q), P.to_device(K), P.to_device(V)
    a = P.GpuCall(w, Qd, Kd, Vd, mu=4, tau=-1.0, variant=oracle.RELAXED)
    b = P.GpuCall(w, Qd, Kd, Vd, mu=23, tau=float("inf"), variant=oracle.RELAXED)
    rows = np.arange(w.B * w.H * w.n_q)
    ra, rb = a.rows(rows), b.rows(rows)
    assert np.array_equal(ra["mixed"].view(np.uint32), rb["mixed"].view(np.uint32))
    assert np.array_equal(ra["out"], rb["out"])


def test_stream_repeated_calls_are_deterministic():
    w = S.Workload(1, 4, 64, 2500, 128, causal=False, seed=14)
    Q, K, V = S.make_qkv(w)
    Qd, Kd, Vd = P.to_device(Q), P.to_device(K), P.to_device(V)
    outs = [lamp.attention(Qd, Kd, Vd, mu=4, tau=0.2, variant=lamp.LAMP_RELAXED, causal=False,
                           want_count=True) for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.out, outs[0].out) and torch.equal(o.mask, outs[0].mask)
        assert o.n_selected.item() == outs[0].n_selected.item()


def test_outlier_4x25x4096_relaxed_sampled():
    w = S.WORKLOADS["outlier_4x25x4096x64"]
    rows = P.sample_rows(w, 6, 5, seed=15)
    run_case(w, 4, 0.3, oracle.RELAXED, rows=rows)


@pytest.mark.parametrize("n_q,variant", [
    (20, oracle.STRICT),      # two streamed passes over the score slab
    (20, oracle.GIVEN_MASK),  # one streamed pass with a caller-given mask
    (3, oracle.STRICT),       # decode rows: the keys split over chunks
])
def test_rows_of_seventy_thousand_keys(n_q, variant):
    """Rows far longer than shared memory (70037 keys) on every path that takes them."""
    n_k = 70037
    w = S.Workload(1, 1, n_q, n_k, 64, causal=True, seed=16 + n_q)
    mask = None
    if variant == oracle.GIVEN_MASK:
        rng = np.random.default_rng(16)
        nv = np.array([w.valid_keys(i) for i in range(w.n_q)])
        mask = S.random_control_mask(w, rng.integers(0, nv // 50 + 1)[None, :]).reshape(1, 1, n_q, -1)
    g, orc, _ = run_case(w, 4, 2e-4, variant, mask_in=mask)  # z is about 1/4600 at the row maximum
    assert g.count() == int(orc.nsel.sum()) > 0


def test_score_slab_limit_is_reported_before_any_launch():
    """A strict problem whose two-pass score slab (B*H*n_q*ceil(n_k/512)*512*4
    bytes) would pass LAMP_MAX_SCORE_SLAB_BYTES fails with LAMP_ERR_UNSUPPORTED
    at planning time (the fake pointers are never used), and its workspace size
    reads 0; the relaxed variant streams the same rows in one pass."""
    fake = 1 << 20
    dims = (1, 32, 16384, 65536, 64)  # 137 GB of slab
    assert 32 * 16384 * 65536 * 4 > lamp.LAMP_MAX_SCORE_SLAB_BYTES
    rc = lamp.lamp_attention_ex(dims=dims, Q=fake, K=fake, V=fake, out=fake, mu=4, tau=0.05,
                                variant=lamp.LAMP_STRICT, causal=1, check=False)
    assert rc == lamp.LAMP_ERR_UNSUPPORTED and "LAMP_MAX_SCORE_SLAB_BYTES" in lamp.lamp_last_error()
    assert lamp.lamp_workspace_size(dims, lamp.LAMP_STRICT) == 0
    assert lamp.lamp_workspace_size(dims, lamp.LAMP_RELAXED) > 0
    # the 16K-token long-context shape (34 GB of slab) is within the limit
    assert lamp.lamp_workspace_size((1, 32, 16384, 16384, 128), lamp.LAMP_STRICT) > 32 * 16384 * 16384 * 4

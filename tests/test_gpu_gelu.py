"""GPU parity of LAMP GELU(scale * x W^T) (GELU after a PS(mu) linear map, the
outputs with condition number kappa > tau recomputed in binary32) against the
CPU oracle, through the C ABI.

Bars:
  * PS(mu) pre-activations and mixed pre-activations: bit-exact.
  * mask: bit-exact, except outputs whose oracle kappa lies within 1e-6 relative
    of tau; those may differ and must number at most 1e-5 of the outputs compared.
  * out_f32 (binary32 GELU on the GPU) within 1e-6 * max(1, |y|) of the oracle's
    double GELU of the same y; bf16 out within one bf16 ulp of the oracle value
    plus that bar.
Shapes put M, N and K on, one past and one short of the 64 x 128 tile and the
32-dimension slice.
"""
import json
import os

import numpy as np
import pytest
import torch

import mixed_precision_attention_ps_b200 as lamp
import oracle
import synthetic as S
from tests import parity as P

pytestmark = pytest.mark.gpu

TAU_FILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tau.json")


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lamp.load()


def golden_tau(name, rate, mu=4):
    for e in json.load(open(TAU_FILE))["entries"]:
        if e["workload"] == name and e["mu"] == mu and e["rate"] == rate:
            return e
    raise KeyError(name)


class GeluRun:
    def __init__(self, x, W, *, mu, tau, variant=oracle.STRICT, scale=1.0, mask_in=None):
        self.M, self.N = x.shape[0], W.shape[0]
        md = None if mask_in is None else torch.from_numpy(np.ascontiguousarray(mask_in).view(np.int32)).cuda()
        self.res = lamp.linear_gelu(P.to_device(x), P.to_device(W), mu=mu, tau=tau, variant=variant, scale=scale,
                                    mask_in=md, want_mask=True, want_out_f32=True, want_scores=True,
                                    want_count=True)
        torch.cuda.synchronize()

    def rows(self, rows):
        r = torch.from_numpy(np.asarray(rows, dtype=np.int64)).cuda()
        take = lambda t: t.index_select(0, r).cpu().numpy()  # noqa: E731
        return {"out": take(self.res.out.view(torch.int16)).view(np.uint16), "out_f32": take(self.res.out_f32),
                "mask": take(self.res.mask).view(np.uint32), "ps": take(self.res.ps),
                "mixed": take(self.res.mixed)}

    def count(self):
        return int(self.res.n_selected.item())


def compare(g, orc, rows, tau, variant):
    """Element-by-element comparison of the GPU rows with the oracle's."""
    N = g["ps"].shape[1]
    assert np.array_equal(g["ps"].view(np.uint32), orc.ps.view(np.uint32)), "PS(mu) outputs differ"
    gb = S.unpack_mask(g["mask"], N)
    ob = S.unpack_mask(orc.mask, N)
    diff = gb != ob
    if diff.any():
        assert variant == oracle.STRICT, "given-mask bits must be copied exactly"
        k = orc.kappa[diff]
        assert np.all(np.abs(k - tau) <= 1e-6 * abs(tau)), "mask differs away from tau"
        assert diff.sum() <= 1e-5 * gb.size
    pad = np.arange(g["mask"].shape[1] * 32) >= N
    assert not np.any(np.unpackbits(g["mask"].view(np.uint8), axis=1, bitorder="little")[:, pad]), "padding bits"
    same = ~diff
    assert np.array_equal(g["mixed"][same].view(np.uint32), orc.mixed[same].view(np.uint32)), "mixed differ"
    y = g["mixed"][same].astype(np.float64)
    o = orc.out[same]
    f = g["out_f32"][same].astype(np.float64)
    fin = np.isfinite(o)
    assert np.array_equal(np.isnan(f), np.isnan(o))
    assert np.all(np.abs(f[fin] - o[fin]) <= 1e-6 * np.maximum(1.0, np.abs(y[fin]))), "out_f32 outside 1e-6"
    # bf16 out: the rounding of a binary32 value within the out_f32 bar
    ob16 = S.bf16_bits_to_f32(S.to_bf16_bits(o)).astype(np.float64)
    gb16 = S.bf16_bits_to_f32(g["out"][same]).astype(np.float64)
    fin = np.isfinite(ob16)
    err = np.abs(gb16[fin] - ob16[fin])
    bar = P.bf16_ulp(ob16[fin]) + 1e-6 * np.maximum(1.0, np.abs(y[fin]))
    i = int(np.argmax(err - bar)) if err.size else 0
    assert np.all(err <= bar), f"bf16 out {gb16[fin][i]} vs oracle {o[fin][i]} (y = {y[fin][i]})"
    return int(gb.sum())


def run_case(lw, mu, tau, variant=oracle.STRICT, mask_in=None, rows=None, x=None, W=None, scale=None):
    if x is None:
        x, W = S.make_linear(lw)
    scale = lw.scale if scale is None else scale
    g = GeluRun(x, W, mu=mu, tau=tau, variant=variant, scale=scale, mask_in=mask_in)
    if rows is None:
        rows = np.arange(x.shape[0], dtype=np.int64)
    orc = oracle.linear_gelu_rows(x, W, scale=scale, mu=mu, tau=tau, variant=variant, mask_in=mask_in,
                                  rows=rows, threads=8)
    nsel = compare(g.rows(rows), orc, rows, tau, variant)
    return g, orc, nsel


@pytest.mark.parametrize("M,N,K", [
    (1, 1, 8),         # one output, one 8-dimension group
    (5, 7, 16),        # below one tile in every direction
    (64, 128, 32),     # exactly one tile and one slice
    (65, 129, 40),     # one past the tile on M and N, a 8-dimension last slice
    (63, 127, 56),     # one short of the tile
    (130, 300, 200),   # several tiles, ragged on all sides
    (3, 1000, 1600),   # deep K (GPT-2 XL's width)
])
def test_gelu_shapes(M, N, K):
    lw = S.LinearWorkload(M, N, K, seed=M + N + K)
    g, orc, nsel = run_case(lw, 4, 2.0)
    assert g.count() == nsel == int(orc.nsel.sum())


@pytest.mark.parametrize("mu", [1, 4, 7, 10, 11, 16, 23])
def test_gelu_rounding_classes(mu):
    lw = S.LinearWorkload(70, 200, 96, seed=500 + mu)
    run_case(lw, mu, 1.5)


@pytest.mark.parametrize("tau", [-1.0, 0.0, 1.0, 4.0, float("inf")])
def test_gelu_threshold_special_cases(tau):
    lw = S.LinearWorkload(40, 150, 64, seed=51)
    g, orc, nsel = run_case(lw, 4, tau)
    if tau < 0:
        assert g.count() == lw.outputs()
    if tau == float("inf"):
        assert g.count() == 0


def test_gelu_calibrated_small_workload():
    lw = S.LINEAR_WORKLOADS["gelu_small_96x300x200"]
    e = golden_tau("gelu_small_96x300x200", 0.016)
    g, orc, nsel = run_case(lw, 4, e["tau"])
    assert g.count() == e["selected_at_tau"]


def test_gelu_given_mask_with_junk_bits():
    lw = S.LinearWorkload(50, 333, 48, seed=52)
    rng = np.random.default_rng(52)
    counts = rng.integers(0, 40, size=lw.M)
    mask = S.linear_random_mask(lw, counts)
    mask[:, -1] |= np.uint32((0xFFFFFFFF << (lw.N % 32)) & 0xFFFFFFFF)  # bits past N: ignored
    g, orc, nsel = run_case(lw, 4, 0.0, variant=oracle.GIVEN_MASK, mask_in=mask)
    assert g.count() == int(counts.sum())


def test_gelu_all_recomputed_equals_mu23():
    lw = S.LinearWorkload(33, 170, 72, seed=53)
    x, W = S.make_linear(lw)
    a = GeluRun(x, W, mu=4, tau=-1.0, scale=lw.scale)
    b = GeluRun(x, W, mu=23, tau=float("inf"), scale=lw.scale)
    rows = np.arange(lw.M)
    ra, rb = a.rows(rows), b.rows(rows)
    assert np.array_equal(ra["mixed"].view(np.uint32), rb["mixed"].view(np.uint32))
    assert np.array_equal(ra["out"], rb["out"])


def test_gelu_extreme_inputs_take_the_exact_path():
    """Tiles whose magnitudes leave the two-instruction rounding's domain (huge or
    subnormal-range products) are computed again with the exact rounding."""
    lw = S.LinearWorkload(128, 256, 64, seed=54)
    x, W = S.make_linear(lw)
    xf, wf = S.bf16_bits_to_f32(x).astype(np.float64), S.bf16_bits_to_f32(W).astype(np.float64)
    xf[:64] *= 2.0 ** 50      # huge products in the first row tile
    wf[:128] *= 2.0 ** 50
    xf[64:] *= 2.0 ** -70     # products below the normal range in the second
    wf[128:] *= 2.0 ** -70
    x2 = S.to_bf16_bits(xf.reshape(-1)).reshape(x.shape)
    W2 = S.to_bf16_bits(wf.reshape(-1)).reshape(W.shape)
    for mu in (4, 10, 23):
        run_case(lw, mu, 2.0, x=x2, W=W2, scale=1.0)


def test_gelu_repeated_calls_are_deterministic():
    lw = S.LinearWorkload(200, 500, 128, seed=55)
    x, W = S.make_linear(lw)
    xd, Wd = P.to_device(x), P.to_device(W)
    outs = [lamp.linear_gelu(xd, Wd, mu=4, tau=2.0, scale=lw.scale, want_count=True) for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.out, outs[0].out) and torch.equal(o.mask, outs[0].mask)
        assert o.n_selected.item() == outs[0].n_selected.item()


@pytest.mark.parametrize("rate", [0.003, 0.016, 0.076])
def test_gelu_gpt2xl_fc_sampled(rate):
    """GPT-2 XL's first MLP layer on 1024 tokens at the calibrated thresholds:
    sampled rows element by element, and the whole call's count equals the
    oracle's count at that tau."""
    name = "gelu_gpt2xl_fc_1024x6400x1600"
    lw = S.LINEAR_WORKLOADS[name]
    e = golden_tau(name, rate)
    rows = np.sort(np.random.default_rng(56).choice(lw.M, size=12, replace=False))
    g, orc, nsel = run_case(lw, 4, e["tau"], rows=rows)
    assert g.count() == e["selected_at_tau"]


def test_gelu_rows_on_both_sides_of_the_tile_split():
    """800 tiles of 128 columns: two full rounds of 128-wide tiles, the rest as
    64-wide tiles in a second launch. Rows from both, and from the row tile
    that the split cuts (row tile 11: columns below and above 5376)."""
    lw = S.LinearWorkload(1024, 6400, 64, seed=57)
    rows = np.array([0, 703, 704, 705, 767, 768, 1000, 1023])
    g, orc, nsel = run_case(lw, 4, 2.0, rows=rows)
    assert nsel > 0


def test_gelu_width_whose_narrow_tiles_do_not_pair():
    """N = 6304: 50 column tiles of 128 but 99 of 64, so no split launch; the
    last wide tile is a quarter full. Sampled rows."""
    lw = S.LinearWorkload(1024, 6304, 32, seed=58)
    rows = np.array([0, 511, 767, 1023])
    g, orc, nsel = run_case(lw, 4, 2.0, rows=rows)
    assert nsel > 0

"""GPU parity of LAMP LayerNorm(scale * x W^T) (LayerNorm after a PS(mu) linear
map; per row the largest magnitudes recomputed in binary32 until the rest meets
the bound) against the CPU oracle, through the C ABI.

Bars:
  * PS(mu) and mixed pre-normalisation rows: bit-exact.
  * mask: bit-exact, except rows where tau lies within 1e-9 relative of one of
    the oracle's threshold values (the row statistics are summed in another
    order on the GPU); such rows must be at most 1e-5 of the rows compared.
  * out_f32 within 1e-6 * max(1, |out|) of the oracle's double LayerNorm; bf16
    out within one bf16 ulp of the oracle value plus that bar.
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


class LnRun:
    def __init__(self, x, W, *, mu, tau, variant=oracle.STRICT, scale=1.0, mask_in=None):
        md = None if mask_in is None else torch.from_numpy(np.ascontiguousarray(mask_in).view(np.int32)).cuda()
        self.res = lamp.linear_layernorm(P.to_device(x), P.to_device(W), mu=mu, tau=tau, variant=variant,
                                         scale=scale, mask_in=md, want_mask=True, want_out_f32=True,
                                         want_scores=True, want_count=True)
        torch.cuda.synchronize()

    def rows(self, rows):
        r = torch.from_numpy(np.asarray(rows, dtype=np.int64)).cuda()
        take = lambda t: t.index_select(0, r).cpu().numpy()  # noqa: E731
        return {"out": take(self.res.out.view(torch.int16)).view(np.uint16), "out_f32": take(self.res.out_f32),
                "mask": take(self.res.mask).view(np.uint32), "ps": take(self.res.ps),
                "mixed": take(self.res.mixed)}

    def count(self):
        return int(self.res.n_selected.item())


def compare(g, orc, tau, variant):
    N = g["ps"].shape[1]
    assert np.array_equal(g["ps"].view(np.uint32), orc.ps.view(np.uint32)), "PS(mu) rows differ"
    gb, ob = S.unpack_mask(g["mask"], N), S.unpack_mask(orc.mask, N)
    bad = np.nonzero((gb != ob).any(axis=1))[0]
    for r in bad:
        assert variant == oracle.STRICT, "given-mask bits must be copied exactly"
        t = oracle.ln_thresholds(orc.ps[r])
        assert np.min(np.abs(t - tau)) <= 1e-9 * abs(tau), f"row {r}: selection differs away from tau"
    assert bad.size <= max(0, int(1e-5 * gb.shape[0])), "too many near-tie rows"
    pad = np.arange(g["mask"].shape[1] * 32) >= N
    assert not np.any(np.unpackbits(g["mask"].view(np.uint8), axis=1, bitorder="little")[:, pad]), "padding bits"
    ok = np.ones(gb.shape[0], bool)
    ok[bad] = False
    assert np.array_equal(g["mixed"][ok].view(np.uint32), orc.mixed[ok].view(np.uint32)), "mixed rows differ"
    o, f = orc.out[ok], g["out_f32"][ok].astype(np.float64)
    bar = 1e-6 * np.maximum(1.0, np.abs(o))
    i = np.unravel_index(int(np.argmax(np.abs(f - o) - bar)), o.shape) if o.size else None
    assert np.all(np.abs(f - o) <= bar), f"out_f32 {f[i]} vs oracle {o[i]}"
    ob16 = S.bf16_bits_to_f32(S.to_bf16_bits(o.reshape(-1))).astype(np.float64).reshape(o.shape)
    gb16 = S.bf16_bits_to_f32(g["out"][ok]).astype(np.float64)
    assert np.all(np.abs(gb16 - ob16) <= P.bf16_ulp(ob16) + bar), "bf16 out beyond one ulp"
    return int(gb.sum())


def run_case(lw, mu, tau, variant=oracle.STRICT, mask_in=None, rows=None):
    x, W = S.make_linear(lw)
    g = LnRun(x, W, mu=mu, tau=tau, variant=variant, scale=lw.scale, mask_in=mask_in)
    if rows is None:
        rows = np.arange(lw.M, dtype=np.int64)
    orc = oracle.linear_ln_rows(x, W, scale=lw.scale, mu=mu, tau=tau, variant=variant, mask_in=mask_in,
                                rows=rows, threads=8)
    nsel = compare(g.rows(rows), orc, tau, variant)
    return g, orc, nsel


@pytest.mark.parametrize("M,N,K", [
    (1, 1, 8),          # one output: LayerNorm of a single value
    (9, 33, 8),         # one past a mask word
    (5, 7, 16),
    (64, 128, 32),      # one tile of the linear map
    (65, 129, 40),      # one past the tile
    (130, 300, 200),
    (3, 1600, 1600),    # GPT-2 XL width
    (6, 8192, 64),      # the longest row
])
def test_ln_shapes(M, N, K):
    lw = S.LinearWorkload(M, N, K, seed=M + N + K + 1)
    tau = 0.8 * np.sqrt(N)  # a few per cent of the largest magnitudes
    g, orc, nsel = run_case(lw, 4, tau)
    assert g.count() == nsel == int(orc.nsel.sum())


@pytest.mark.parametrize("mu", [1, 4, 7, 10, 11, 16, 23])
def test_ln_rounding_classes(mu):
    lw = S.LinearWorkload(40, 200, 96, seed=600 + mu)
    run_case(lw, mu, 10.0)


@pytest.mark.parametrize("tau", [-1.0, 0.0, 5.0, float("inf")])
def test_ln_threshold_special_cases(tau):
    lw = S.LinearWorkload(30, 250, 64, seed=61)
    g, orc, nsel = run_case(lw, 4, tau)
    if tau < 0:
        assert g.count() == lw.outputs()
    if tau == float("inf"):
        assert g.count() == 0


def test_ln_calibrated_small_workload():
    lw = S.LINEAR_WORKLOADS["ln_small_64x300x128"]
    e = golden_tau("ln_small_64x300x128", 0.016)
    g, orc, nsel = run_case(lw, 4, e["tau"])
    assert g.count() == e["selected_at_tau"]


def test_ln_given_mask_with_junk_bits():
    lw = S.LinearWorkload(40, 301, 48, seed=62)
    rng = np.random.default_rng(62)
    counts = rng.integers(0, 30, size=lw.M)
    mask = S.linear_random_mask(lw, counts)
    mask[:, -1] |= np.uint32((0xFFFFFFFF << (lw.N % 32)) & 0xFFFFFFFF)  # bits past N: ignored
    g, orc, nsel = run_case(lw, 4, 0.0, variant=oracle.GIVEN_MASK, mask_in=mask)
    assert g.count() == int(counts.sum())


def test_ln_all_recomputed_equals_mu23():
    lw = S.LinearWorkload(20, 400, 72, seed=63)
    x, W = S.make_linear(lw)
    a = LnRun(x, W, mu=4, tau=-1.0, scale=lw.scale)
    b = LnRun(x, W, mu=23, tau=float("inf"), scale=lw.scale)
    rows = np.arange(lw.M)
    ra, rb = a.rows(rows), b.rows(rows)
    assert np.array_equal(ra["mixed"].view(np.uint32), rb["mixed"].view(np.uint32))
    assert np.array_equal(ra["out"], rb["out"])


def test_ln_scratch_from_the_pool_and_from_the_caller():
    """y_hat in ps_out, in the library's pool, or in a caller workspace: the same outputs."""
    lw = S.LinearWorkload(50, 700, 64, seed=64)
    x, W = S.make_linear(lw)
    xd, Wd = P.to_device(x), P.to_device(W)
    a = lamp.linear_layernorm(xd, Wd, mu=4, tau=15.0, scale=lw.scale, want_scores=True)
    b = lamp.linear_layernorm(xd, Wd, mu=4, tau=15.0, scale=lw.scale)
    out = torch.empty_like(a.out)
    mask = torch.empty_like(a.mask)
    nbytes = lamp.lamp_ln_workspace_size(lw.M, lw.N)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    lamp.lamp_linear_layernorm(M=lw.M, N=lw.N, K=lw.K, x=xd, W=Wd, out=out, mask_out=mask, mu=4, tau=15.0,
                               scale=lw.scale, workspace=ws, workspace_bytes=nbytes,
                               stream=torch.cuda.current_stream())
    torch.cuda.synchronize()
    for r in (b, ):
        assert torch.equal(r.out, a.out) and torch.equal(r.mask, a.mask)
    assert torch.equal(out, a.out) and torch.equal(mask, a.mask)


def test_ln_repeated_calls_are_deterministic():
    lw = S.LinearWorkload(100, 1600, 128, seed=65)
    x, W = S.make_linear(lw)
    xd, Wd = P.to_device(x), P.to_device(W)
    outs = [lamp.linear_layernorm(xd, Wd, mu=4, tau=30.0, scale=lw.scale, want_count=True) for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.out, outs[0].out) and torch.equal(o.mask, outs[0].mask)
        assert o.n_selected.item() == outs[0].n_selected.item()


@pytest.mark.parametrize("rate", [0.003, 0.016, 0.076])
def test_ln_gpt2xl_proj_sampled(rate):
    """GPT-2 XL's attention output projection on 1024 tokens at the calibrated
    thresholds: sampled rows element by element, the whole call's count equal
    to the oracle's."""
    name = "ln_gpt2xl_proj_1024x1600x1600"
    lw = S.LINEAR_WORKLOADS[name]
    e = golden_tau(name, rate)
    rows = np.sort(np.random.default_rng(66).choice(lw.M, size=24, replace=False))
    g, orc, nsel = run_case(lw, 4, e["tau"], rows=rows)
    assert g.count() == e["selected_at_tau"]


def test_ln_wide_tiles_of_the_linear_map():
    """A shape whose linear map takes the 128-wide tiles (800 of them) and rows of
    6400 outputs; sampled rows."""
    lw = S.LinearWorkload(1024, 6400, 64, seed=67)
    rows = np.array([0, 1, 63, 64, 500, 1023])
    g, orc, nsel = run_case(lw, 4, 72.0, rows=rows)
    assert 0 < nsel

"""PS(mu) rounding of the oracle, pinned to definitions outside the oracle.

PS(mu) is the simulated format of the LAMP summary, "Experimental results"
(mu mantissa bits); the reading (binary32 exponent range and subnormals, round
to nearest with ties to even) is the one the oracle header states.
"""
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "round_ps.txt")


def grid_nearest(x32: np.ndarray, mu: int) -> np.ndarray:
    """Nearest value of the PS(mu) grid, ties to even, computed in double."""
    x = x32.astype(np.float64)
    out = x.copy()
    fin = np.isfinite(x) & (x != 0)
    ax = np.abs(x[fin])
    _, ex = np.frexp(ax)
    E = np.maximum(ex - 1, -126)
    q = np.ldexp(1.0, E - mu)
    r = np.rint(ax / q) * q
    r[r >= 2.0 ** 128] = np.inf
    out[fin] = np.sign(x[fin]) * r
    return out.astype(np.float32)


def structured_sample(mu: int, seed: int = 1) -> np.ndarray:
    """Every exponent field, with fraction patterns around the rounding position
    (exact ties, one ulp either side, all-ones, random) and random patterns."""
    s = 23 - mu
    rng = np.random.default_rng(seed)
    fr = [0, 1, (1 << 23) - 1]
    if s > 0:
        half = 1 << (s - 1)
        for kept in [0, 1, 2, 3, (1 << mu) - 1 if mu > 0 else 0, (1 << mu) - 2 if mu > 1 else 0]:
            base = (kept << s) & ((1 << 23) - 1)
            fr += [base | half, (base | half) + 1, (base | half) - 1, base, base | (half - 1 if half > 1 else 0)]
    fr += list(rng.integers(0, 1 << 23, 64))
    fr = np.array(sorted(set(int(f) & ((1 << 23) - 1) for f in fr)), dtype=np.uint32)
    exps = np.arange(256, dtype=np.uint32)
    pats = (exps[:, None] << np.uint32(23)) | fr[None, :]
    pats = np.concatenate([pats.reshape(-1), pats.reshape(-1) | np.uint32(0x80000000),
                           rng.integers(0, 2 ** 32, 200000, dtype=np.uint64).astype(np.uint32)])
    return pats.view(np.float32)


def _bits(a):
    return np.asarray(a, dtype=np.float32).view(np.uint32)


def test_golden_hand_cases():
    n = 0
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if not line:
            continue
        mu, x, want = line.split()
        x = np.array([int(x, 16)], dtype=np.uint32).view(np.float32)
        got = oracle.round_ps(x, int(mu))
        assert _bits(got)[0] == int(want, 16), (mu, hex(_bits(x)[0]), hex(_bits(got)[0]), want)
        n += 1
    assert n >= 20


@pytest.mark.parametrize("mu", [1, 2, 4, 6, 7, 10, 11, 16, 21, 22])
def test_matches_grid_nearest_on_structured_sample(mu):
    x = structured_sample(mu)
    got = oracle.round_ps(x, mu)
    want = grid_nearest(x, mu)
    nan = np.isnan(x)
    assert np.array_equal(_bits(got)[~nan], _bits(want)[~nan])
    assert np.array_equal(_bits(got)[nan], _bits(x)[nan])


def test_mu23_is_identity():
    x = structured_sample(23)
    assert np.array_equal(_bits(oracle.round_ps(x, 23)), _bits(x))


def test_mu7_equals_binary32_to_bfloat16():
    """mu = 7 is bfloat16's fraction width with binary32's exponent range, so the
    rounding must equal torch's float32 -> bfloat16 conversion (round to nearest even)."""
    x = structured_sample(7, seed=3)
    x = x[np.isfinite(x)]
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).to(torch.float32).numpy()
    got = oracle.round_ps(x, 7)
    assert np.array_equal(_bits(got), _bits(want))


def test_rounding_is_idempotent_and_monotone():
    rng = np.random.default_rng(5)
    x = np.sort(rng.standard_normal(100000).astype(np.float32) * 10)
    for mu in (3, 4, 10):
        r = oracle.round_ps(x, mu)
        assert np.array_equal(_bits(oracle.round_ps(r, mu)), _bits(r))
        assert np.all(np.diff(r.astype(np.float64)) >= 0)
        # error within half a unit of the mu-bit grid
        err = np.abs(r.astype(np.float64) - x.astype(np.float64))
        assert np.all(err <= np.ldexp(np.abs(x.astype(np.float64)), -(mu + 1)) * (1 + 1e-12))


@pytest.mark.parametrize("mu", [4, 10])
def test_exhaustive_all_binary32_patterns(mu, tmp_path):
    """All 2^32 bit patterns against the grid definition (C, OpenMP)."""
    lib = oracle.build()
    exe = tmp_path / "exhaustive_round"
    src = os.path.join(os.path.dirname(__file__), "exhaustive_round.c")
    subprocess.run(["gcc", "-O2", "-fopenmp", src, "-o", str(exe), lib, "-lm",
                    f"-Wl,-rpath,{os.path.dirname(lib)}"], check=True)
    out = subprocess.run([str(exe), str(mu)], check=True, capture_output=True, text=True)
    assert int(out.stdout.strip()) == 0

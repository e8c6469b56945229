"""Helpers of the GPU parity tests: run the CUDA path through the C ABI on seeded
synthetic inputs and compare it with the CPU oracle element by element.

Bars (the numerical contract of include/lamp.h):
  * PS(mu) scores, FP32-recomputed (mixed) scores: bit-exact.
  * mask: bit-exact, except entries whose oracle criterion lies within 1e-6
    relative of tau; those may differ and must number at most 1e-5 of the
    valid entries compared.
  * out_f32 within 2e-3 (absolute) of the oracle's double-precision output;
    bf16 out within max(2e-3, one bf16 ulp of the oracle value).
  * row KL(P_oracle || P_gpu) < 1e-6, with P_gpu = exp(mixed - lse) rebuilt
    from the GPU's mixed scores and log-sum-exp (generalised KL, since that P_gpu
    sums to one only up to the GPU's rounding of lse).
"""
from __future__ import annotations

import numpy as np
import torch

import mixed_precision_attention_ps_b200 as lamp
import oracle
import synthetic as S

OUT_F32_TOL = 2e-3
KL_TOL = 1e-6
TIE_REL = 1e-6
TIE_FRAC = 1e-5

# (label, near-tie mask differences, valid entries compared) of the calibrated-tau
# cases, summarised at the end of the test session (tests/conftest.py)
TIE_LOG: list = []


def to_device(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


class GpuCall:
    """One call of lamp_attention_ex with every optional output switched on."""

    def __init__(self, w: S.Workload, Qd, Kd, Vd, *, mu, tau, variant, mask_in=None, scale=0.0,
                 want_scores=True):
        res = lamp.attention(Qd, Kd, Vd, mu=mu, tau=tau, variant=variant, causal=w.causal, scale=scale,
                             mask_in=mask_in, want_mask=True, want_out_f32=True, want_scores=want_scores,
                             want_lse=True, want_count=True)
        torch.cuda.synchronize()
        self.res = res
        self.w = w

    def rows(self, rows: np.ndarray) -> dict:
        w = self.w
        r = torch.from_numpy(np.asarray(rows, dtype=np.int64)).cuda()
        B, H, n_q = w.B, w.H, w.n_q

        def take(t, width):
            return t.reshape(B * H * n_q, width).index_select(0, r).cpu().numpy()

        d = {
            "out": take(self.res.out.view(torch.int16), w.d).view(np.uint16),
            "out_f32": take(self.res.out_f32, w.d),
            "mask": take(self.res.mask, (w.n_k + 31) // 32).view(np.uint32),
            "lse": take(self.res.lse, 1)[:, 0],
        }
        if self.res.ps_scores is not None:
            d["ps"] = take(self.res.ps_scores, w.n_k)
            d["mixed"] = take(self.res.mixed_scores, w.n_k)
        return d

    def count(self) -> int:
        return int(self.res.n_selected.item())


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x).astype(np.float64)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def row_valid(w: S.Workload, rows: np.ndarray) -> np.ndarray:
    return np.array([w.valid_keys(int(r) % w.n_q) for r in rows], dtype=np.int64)


def compare(w: S.Workload, gpu: dict, orc: oracle.RowResult, rows: np.ndarray, tau: float,
            variant: int, check_scores: bool = True) -> dict:
    """Assert every bar; return a few statistics for the test log."""
    nv = row_valid(w, rows)
    stats = {"rows": len(rows), "valid": int(nv.sum())}
    # --- mask, with the near-tie allowance ------------------------------------
    gm = S.unpack_mask(gpu["mask"], w.n_k)
    om = S.unpack_mask(orc.mask, w.n_k)
    diff = gm != om
    # padding words past n_k must be zero as well
    nwords = (w.n_k + 31) // 32
    if w.n_k % 32:
        assert np.all(gpu["mask"][:, nwords - 1] >> np.uint32(w.n_k % 32) == 0)
    ties = 0
    if diff.any():
        assert variant != oracle.GIVEN_MASK, "given-mask selection must be exact"
        assert orc.crit is not None, "mask differs; rerun the oracle with want_crit for the tie check"
        ri, ji = np.nonzero(diff)
        c = orc.crit[ri, ji]
        near = np.abs(c - tau) <= TIE_REL * abs(tau)
        assert near.all(), f"mask mismatch away from tau at rows {rows[ri[~near]][:5]} keys {ji[~near][:5]}"
        ties = int(diff.sum())
        assert ties <= max(1, int(TIE_FRAC * nv.sum())), f"{ties} near-tie mask mismatches"
    stats["ties"] = ties
    # --- scores -----------------------------------------------------------------
    if check_scores and "ps" in gpu:
        assert np.array_equal(gpu["ps"].view(np.uint32), orc.ps.view(np.uint32)), _first_diff(gpu["ps"], orc.ps)
        ok = ~diff
        gmix, omix = gpu["mixed"], orc.mixed
        assert np.array_equal(gmix.view(np.uint32)[ok], omix.view(np.uint32)[ok]), _first_diff(gmix, omix)
        # where a near tie flipped, the GPU must hold the other legitimate value
        if diff.any():
            y32 = orc.y32
            ri, ji = np.nonzero(diff)
            want = np.where(gm[ri, ji], y32[ri, ji], orc.ps[ri, ji])
            assert np.array_equal(gmix[ri, ji].view(np.uint32), want.view(np.uint32))
    # --- outputs ------------------------------------------------------------------
    err32 = np.abs(gpu["out_f32"].astype(np.float64) - orc.out)
    stats["max_abs_f32"] = float(err32.max()) if err32.size else 0.0
    assert stats["max_abs_f32"] <= OUT_F32_TOL, stats
    outb = S.bf16_bits_to_f32(gpu["out"]).astype(np.float64)
    errb = np.abs(outb - orc.out)
    tolb = np.maximum(OUT_F32_TOL, bf16_ulp(orc.out))
    stats["max_abs_bf16"] = float(errb.max()) if errb.size else 0.0
    assert np.all(errb <= tolb), stats
    # empty rows: out = 0, lse = -inf
    empty = nv == 0
    if empty.any():
        assert np.all(gpu["out_f32"][empty] == 0) and np.all(np.isneginf(gpu["lse"][empty]))
    lse_err = np.abs(gpu["lse"][~empty].astype(np.float64) - orc.lse[~empty])
    assert np.all(lse_err <= 1e-5 * np.maximum(1.0, np.abs(orc.lse[~empty]))), lse_err.max()
    # --- row KL of the probabilities ------------------------------------------------
    if "mixed" in gpu:
        kls = []
        for t in np.nonzero(~empty)[0]:
            n = nv[t]
            lp = orc.mixed[t, :n].astype(np.float64) - orc.lse[t]
            lq = gpu["mixed"][t, :n].astype(np.float64) - float(gpu["lse"][t])
            p, q = np.exp(lp), np.exp(lq)
            # generalised KL (q need not sum to exactly one): sum p log(p/q) - sum p + sum q
            kls.append(float(np.sum(p * (lp - lq)) - p.sum() + q.sum()))
        stats["max_row_kl"] = max(kls) if kls else 0.0
        assert stats["max_row_kl"] < KL_TOL, stats
    return stats


def _first_diff(a, b):
    ua, ub = a.view(np.uint32), b.view(np.uint32)
    idx = np.argwhere(ua != ub)
    if idx.size == 0:
        return "equal"
    r, j = idx[0]
    return f"{len(idx)} differences; first at row {r} key {j}: gpu {a[r, j]!r} oracle {b[r, j]!r}"


def sample_rows(w: S.Workload, n_per_head: int, n_heads: int, seed: int = 0) -> np.ndarray:
    """Flat row ids: the first and last rows and random ones, over a spread of heads."""
    rng = np.random.default_rng(seed)
    BH = w.B * w.H
    heads = np.unique(np.concatenate([[0, BH - 1], rng.integers(0, BH, max(0, n_heads - 2))]))
    rows = []
    for bh in heads:
        pick = set([0, 1, w.n_q - 1, w.n_q // 2]) | set(rng.integers(0, w.n_q, n_per_head).tolist())
        rows += [bh * w.n_q + i for i in sorted(pick) if 0 <= i < w.n_q]
    return np.array(rows, dtype=np.int64)

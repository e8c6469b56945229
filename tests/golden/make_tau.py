"""Write tests/golden/tau.json: selection thresholds that give the recompute
rates of the experiments, computed with the CPU oracle only.

LAMP summary, "Experimental results": the accuracy figures are quoted at
recompute rates of 0.3 %, 1.6 % and 7.6 % of the key-query products (mu = 4).
For a workload, a variant and mu, tau is the (k+1)-th largest criterion value
over the valid (query, key) entries, k = round(rate * entries); the entries
strictly above it are selected, so the selected count is at most k (fewer when
criterion values tie).

The activation workloads (GELU after a PS(mu) linear map) calibrate on the
condition number kappa_j of every output. Their low-precision outputs take few
distinct values (mu = 4 keeps 5 significant bits), so kappa ties heavily; tau is
put halfway between the (k+1)-th largest value and the next larger distinct one,
which selects the same entries and keeps every kappa far from tau (a last-bit
difference between two exp implementations then decides nothing).

The LayerNorm workloads select per row greedily (the largest magnitudes until
the rest meets the bound); a row's count changes at the oracle's threshold
values sqrt(sum of the m smallest squares) / sigma, so tau is put halfway between
the two consecutive distinct thresholds (over all rows) that give k recomputed
outputs in total.

Entries are taken from the whole workload, except for the 16K-token workload,
where the oracle evaluates a uniform random sample of query rows (seeded; the
row count is recorded). Sampling rows uniformly keeps the entry distribution,
since every entry of a sampled row is counted.

    python tests/golden/make_tau.py [--threads N] [--only NAME]
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synthetic as S  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tau.json")

# (workload, variant, mu list, rates, sampled rows or None)
PLAN = [
    ("gpt2xl_1x25x1024x64", oracle.STRICT, [4, 7, 10], [0.003, 0.016, 0.076], None),
    ("batch8_8x25x1024x64", oracle.RELAXED, [4], [0.016], None),
    ("long_1x32x16384x128", oracle.RELAXED, [4], [0.01], 768),
    ("long_1x8x4096x128", oracle.RELAXED, [4], [0.01], None),
    ("decode_1x32x1x16384x128", oracle.STRICT, [4], [0.016], None),
    ("decode_1x32x1x16384x128", oracle.RELAXED, [4], [0.01], None),
    ("outlier_4x25x4096x64", oracle.STRICT, [4, 6], [0.003, 0.076], None),
    ("gelu_small_96x300x200", oracle.STRICT, [4], [0.016], None),
    ("gelu_gpt2xl_fc_1024x6400x1600", oracle.STRICT, [4], [0.003, 0.016, 0.076], None),
    ("ln_small_64x300x128", oracle.STRICT, [4], [0.016], None),
    ("ln_gpt2xl_proj_1024x1600x1600", oracle.STRICT, [4], [0.003, 0.016, 0.076], None),
]


class TopK:
    """The largest values of a stream, kept to at most `keep` entries."""

    def __init__(self, keep: int):
        self.keep = keep
        self.vals = np.empty(0, np.float64)

    def add(self, v: np.ndarray):
        v = np.concatenate([self.vals, v])
        if v.size > self.keep:
            v = np.partition(v, v.size - self.keep)[v.size - self.keep:]
        self.vals = v

    def kth_largest(self, k: int) -> float:
        """(k+1)-th largest value seen (k counted from 0)."""
        s = np.sort(self.vals)[::-1]
        return float(s[k])


def calibrate_linear(name, mu, rates, threads):
    lw = S.LINEAR_WORKLOADS[name]
    x, W = S.make_linear(lw)
    entries = lw.outputs()
    ks = [int(round(r * entries)) for r in rates]
    top = TopK(max(ks) + 1)
    chunk = max(1, int(2 ** 22 // lw.N))
    for lo in range(0, lw.M, chunk):
        rows = np.arange(lo, min(lw.M, lo + chunk), dtype=np.int64)
        res = oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=mu, tau=np.inf, rows=rows, threads=threads)
        top.add(res.kappa.reshape(-1))
    out = []
    for rate, k in zip(rates, ks):
        v = top.kth_largest(k)
        above = top.vals[top.vals > v]
        tau = 0.5 * (v + float(above.min())) if above.size else v
        out.append({"workload": name, "variant": int(oracle.STRICT), "mu": mu, "rate": rate, "tau": tau,
                    "k": k, "entries": entries, "selected_at_tau": int(np.sum(top.vals > tau)), "rows": "all"})
    return out


def calibrate_ln(name, mu, rates, threads):
    lw = S.LINEAR_WORKLOADS[name]
    x, W = S.make_linear(lw)
    res = oracle.linear_ln_rows(x, W, scale=lw.scale, mu=mu, tau=np.inf, threads=threads)
    t = np.sort(np.concatenate([oracle.ln_thresholds(res.ps[r]) for r in range(lw.M)]))
    entries = lw.outputs()
    out = []
    for rate in rates:
        k = int(round(rate * entries))
        lo = t[entries - k - 1]          # the (entries - k)-th smallest threshold: met
        above = t[t > lo]
        tau = 0.5 * (lo + float(above.min())) if above.size else float(lo)
        sel = int(entries - np.searchsorted(t, tau, side="right"))
        out.append({"workload": name, "variant": int(oracle.STRICT), "mu": mu, "rate": rate, "tau": tau,
                    "k": k, "entries": entries, "selected_at_tau": sel, "rows": "all"})
    return out


def calibrate(name, variant, mu, rates, sample_rows, threads):
    if name.startswith("ln_"):
        return calibrate_ln(name, mu, rates, threads)
    if name in S.LINEAR_WORKLOADS:
        return calibrate_linear(name, mu, rates, threads)
    w = S.WORKLOADS[name]
    Q, K, V = S.make_qkv(w)
    total_rows = w.B * w.H * w.n_q
    if sample_rows:
        rng = np.random.default_rng(12345)
        rows = np.sort(rng.choice(total_rows, size=sample_rows, replace=False)).astype(np.int64)
    else:
        rows = np.arange(total_rows, dtype=np.int64)
    nv = np.array([w.valid_keys(int(r) % w.n_q) for r in rows], dtype=np.int64)
    entries = int(nv.sum())
    ks = [int(round(r * entries)) for r in rates]
    top = TopK(max(ks) + 1)
    chunk = max(1, int(2 ** 25 // w.n_k))
    for lo in range(0, rows.size, chunk):
        sub = rows[lo:lo + chunk]
        res = oracle.attention_rows(Q, K, V, causal=w.causal, mu=mu, tau=np.inf, variant=variant, rows=sub,
                                    want_scores=False, want_crit=True, threads=threads)
        vals = np.concatenate([res.crit[t, :nv[lo + t]] for t in range(sub.size)])
        top.add(vals)
    out = []
    for rate, k in zip(rates, ks):
        tau = top.kth_largest(k)
        count = int(np.sum(top.vals > tau))
        out.append({"workload": name, "variant": int(variant), "mu": mu, "rate": rate, "tau": tau,
                    "k": k, "entries": entries, "selected_at_tau": count,
                    "rows": "all" if not sample_rows else f"{sample_rows} random rows (seed 12345)"})
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--threads", type=int, default=os.cpu_count() or 1)
    ap.add_argument("--only")
    a = ap.parse_args()
    table = []
    if a.only and os.path.exists(OUT):
        table = [e for e in json.load(open(OUT))["entries"] if e["workload"] != a.only]
    for name, variant, mus, rates, sample in PLAN:
        if a.only and name != a.only:
            continue
        for mu in mus:
            t0 = time.time()
            table += calibrate(name, variant, mu, rates, sample, a.threads)
            print(f"{name} variant={variant} mu={mu}: {time.time() - t0:.1f} s", flush=True)
    doc = {
        "source": "LAMP summary (gist.science paper 2601.21623), 'Experimental results': recompute "
                  "rates 0.3/1.6/7.6 % at mu = 4; tau = (k+1)-th largest oracle criterion value",
        "written_by": "tests/golden/make_tau.py (CPU oracle only)",
        "entries": table,
    }
    with open(OUT, "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()

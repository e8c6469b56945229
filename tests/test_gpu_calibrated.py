"""GPU parity at exactly the thresholds the bench runs.

Every attention entry of tests/golden/tau.json (the recompute rates 0.3/1.6/7.6 %
of the LAMP summary's "Experimental results", calibrated on the oracle by
tests/golden/make_tau.py) is run as one full-size call and compared with the
oracle on sampled rows. Both sides receive the binary32 value of the stored tau,
which is what the C ABI (float tau) and bench.py pass, so that the only
mismatches left are the near ties the contract allows (criterion within 1e-6
relative of tau, at most 1e-5 of the entries); their count is logged and
summarised at the end of the session.

The random-selection control of the same section ("random selection of the same
count") runs as LAMP_GIVEN_MASK at the GPT-2 XL and outlier shapes: per row,
floor(rate * valid keys) keys chosen uniformly by synthetic.random_control_mask,
the same mask given to both sides.
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


def attention_entries():
    doc = json.load(open(TAU_FILE))
    return [e for e in doc["entries"] if e["workload"] in S.WORKLOADS]


# rows compared per entry: (rows per head, heads) for sample_rows
SAMPLE = {
    "gpt2xl_1x25x1024x64": (16, 6),
    "batch8_8x25x1024x64": (8, 8),
    "long_1x32x16384x128": (2, 3),
    "long_1x8x4096x128": (6, 4),
    "outlier_4x25x4096x64": (4, 4),
}

_inputs = {}


def inputs(name):
    if name not in _inputs:
        _inputs.clear()  # one workload's device inputs at a time
        w = S.WORKLOADS[name]
        Q, K, V = S.make_qkv(w)
        _inputs[name] = (w, Q, K, V, P.to_device(Q), P.to_device(K), P.to_device(V))
    return _inputs[name]


def run(name, mu, tau, variant, rows, mask_in=None, label=""):
    w, Q, K, V, Qd, Kd, Vd = inputs(name)
    md = None if mask_in is None else torch.from_numpy(np.ascontiguousarray(mask_in).view(np.int32)).cuda()
    g = P.GpuCall(w, Qd, Kd, Vd, mu=mu, tau=tau, variant=variant, mask_in=md)
    orc = oracle.attention_rows(Q, K, V, causal=w.causal, mu=mu, tau=tau, variant=variant, mask_in=mask_in,
                                rows=rows, want_crit=True, threads=8)
    st = P.compare(w, g.rows(rows), orc, rows, tau, variant)
    P.TIE_LOG.append((label, st["ties"], st["valid"]))
    del g
    torch.cuda.empty_cache()
    return st


@pytest.mark.parametrize("e", attention_entries(),
                         ids=lambda e: f"{e['workload']}-v{e['variant']}-mu{e['mu']}-r{e['rate']}")
def test_calibrated_tau(e):
    """The full-size call at a calibrated tau, sampled rows against the oracle."""
    name = e["workload"]
    w = S.WORKLOADS[name]
    tau32 = float(np.float32(e["tau"]))
    if name in SAMPLE:
        rows = P.sample_rows(w, *SAMPLE[name], seed=int(1e4 * e["rate"]) + e["mu"])
    else:  # decode shapes: every row
        rows = np.arange(w.B * w.H * w.n_q, dtype=np.int64)
    st = run(name, e["mu"], tau32, e["variant"], rows,
             label=f"{name} v{e['variant']} mu{e['mu']} rate {e['rate']}")
    print(st)


@pytest.mark.parametrize("name,heads,rate", [
    ("gpt2xl_1x25x1024x64", None, 0.016),
    ("outlier_4x25x4096x64", (0, 37, 99), 0.076),
])
def test_random_control_given_mask(name, heads, rate):
    """The matched-rate random control (LAMP_GIVEN_MASK) at full size: every row of
    the listed heads (all heads when None) gets floor(rate * valid keys) uniformly
    chosen keys, the other heads an empty mask."""
    w = S.WORKLOADS[name]
    BH = w.B * w.H
    heads = list(range(BH)) if heads is None else list(heads)
    nv = np.array([w.valid_keys(i) for i in range(w.n_q)], dtype=np.int64)
    counts = np.floor(rate * nv).astype(np.int64)
    nwords = (w.n_k + 31) // 32
    mask = np.zeros((BH, w.n_q, nwords), dtype=np.uint32)
    mask[heads] = S.random_control_mask(w, np.tile(counts, (len(heads), 1)), bh_list=heads)
    mask = mask.reshape(w.B, w.H, w.n_q, nwords)
    rng = np.random.default_rng(11)
    rows = []
    for bh in heads[:: max(1, len(heads) // 5)]:
        pick = {0, w.n_q - 1} | set(rng.integers(0, w.n_q, 6).tolist())
        rows += [bh * w.n_q + i for i in sorted(pick)]
    rows = np.array(rows, dtype=np.int64)
    st = run(name, 4, 0.0, oracle.GIVEN_MASK, rows, mask_in=mask, label=f"{name} random control {rate}")
    assert st["ties"] == 0
    print(st)

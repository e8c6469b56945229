"""lamp_attention_noalloc: the entry point for callers that must not allocate
device memory (for instance a program whose allocator owns all device memory,
or one that allocates only at start-up). Its scratch is a fixed array in the
library's device memory, shared by every call; this file checks, through the C
ABI, that two calls in a row give exactly the results of lamp_attention_ex (the
same kernels on the same inputs: out, out_f32, lse and the mask bit for bit),
that the shared scratch carries nothing from one call into the next, and that
the call refuses a caller workspace and problems larger than its scratch. The
cases cover the whole-row, streamed and split-key decode kernels (the decode
kernels keep per-row completion counters in the scratch) and a caller-given
mask.

It is collected last (file name), so that a run stopping at the first failure
has already run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import mixed_precision_attention_ps_b200 as lamp
import synthetic as S
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lamp.load()


def outputs(w):
    dev = torch.device("cuda")
    return {
        "out": torch.empty((w.B, w.H, w.n_q, w.d), dtype=torch.bfloat16, device=dev),
        "out_f32": torch.empty((w.B, w.H, w.n_q, w.d), dtype=torch.float32, device=dev),
        "mask": torch.empty((w.B, w.H, w.n_q, (w.n_k + 31) // 32), dtype=torch.int32, device=dev),
        "lse": torch.empty((w.B, w.H, w.n_q), dtype=torch.float32, device=dev),
        "nsel": torch.empty(1, dtype=torch.int64, device=dev),
    }


def call(entry, w, Qd, Kd, Vd, o, mu, tau, variant, **extra):
    entry(dims=(w.B, w.H, w.n_q, w.n_k, w.d), Q=Qd, K=Kd, V=Vd, out=o["out"], mask_out=o["mask"], mu=mu,
          tau=tau, variant=variant, causal=int(w.causal), out_f32=o["out_f32"], lse_out=o["lse"],
          n_selected_out=o["nsel"], **extra)


@pytest.mark.parametrize("w,mu,tau,variant", [
    (S.Workload(1, 3, 300, 300, 64, seed=21), 4, 0.03, lamp.LAMP_STRICT),
    (S.Workload(2, 2, 100, 517, 128, causal=False, seed=22), 6, 0.5, lamp.LAMP_RELAXED),
    (S.Workload(1, 2, 40, 3000, 64, causal=False, seed=23), 4, 0.02, lamp.LAMP_STRICT),
    # relaxed rows longer than 1024 keys: the streamed one-pass kernel
    (S.Workload(1, 2, 40, 2500, 64, causal=False, seed=26), 4, 0.3, lamp.LAMP_RELAXED),
    (S.Workload(1, 1, 24, 1500, 128, seed=27), 6, 0.2, lamp.LAMP_RELAXED),
    # a few query rows against long key rows: the split-key decode kernels
    (S.Workload(1, 4, 2, 4096, 128, seed=28), 4, 0.002, lamp.LAMP_STRICT),
    (S.Workload(1, 4, 2, 4096, 128, seed=29), 4, 1.0, lamp.LAMP_RELAXED),
    # the random control: a caller-given mask
    (S.Workload(1, 2, 90, 200, 64, seed=30), 4, 0.0, lamp.LAMP_GIVEN_MASK),
])
def test_matches_the_allocating_entry_on_two_calls_in_a_row(w, mu, tau, variant):
    Q, K, V = S.make_qkv(w)
    Qd, Kd, Vd = P.to_device(Q), P.to_device(K), P.to_device(V)
    extra = {}
    if variant == lamp.LAMP_GIVEN_MASK:
        nv = np.array([w.valid_keys(i) for i in range(w.n_q)])
        counts = np.tile(nv // 10, (w.B * w.H, 1))
        m = S.random_control_mask(w, counts).reshape(w.B, w.H, w.n_q, -1)
        extra["mask_in"] = torch.from_numpy(m.view(np.int32)).cuda()
    ref = outputs(w)
    dims = (w.B, w.H, w.n_q, w.n_k, w.d)
    need = lamp.lamp_workspace_size(dims, variant)
    assert 0 < need <= lamp.LAMP_NOALLOC_SCRATCH_BYTES
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    call(lamp.lamp_attention_ex, w, Qd, Kd, Vd, ref, mu, tau, variant, workspace=ws, workspace_bytes=need, **extra)
    torch.cuda.synchronize()
    assert ref["nsel"].item() > 0
    for _ in range(2):
        got = outputs(w)
        for t in got.values():  # stale values must not survive into the result
            t.view(torch.uint8).fill_(0xA5)
        call(lamp.lamp_attention_noalloc, w, Qd, Kd, Vd, got, mu, tau, variant, **extra)
        torch.cuda.synchronize()
        for name in ("out", "out_f32", "lse", "mask", "nsel"):  # bit for bit
            assert torch.equal(got[name].view(torch.uint8), ref[name].view(torch.uint8)), name


def test_refuses_a_workspace_and_oversized_problems():
    w = S.Workload(1, 1, 16, 64, 64, seed=24)
    Q, K, V = S.make_qkv(w)
    Qd, Kd, Vd = P.to_device(Q), P.to_device(K), P.to_device(V)
    o = outputs(w)
    ws = torch.empty(1 << 16, dtype=torch.uint8, device="cuda")
    rc = lamp.lamp_attention_noalloc(dims=(1, 1, 16, 64, 64), Q=Qd, K=Kd, V=Vd, out=o["out"], mu=4, tau=0.1,
                                     workspace=ws, workspace_bytes=ws.numel(), check=False)
    assert rc == lamp.LAMP_ERR_ARG and "workspace" in lamp.lamp_last_error()
    # strict rows of 6000 keys in 16 heads take two streamed passes over a score
    # slab of 16 * 32 * 6144 * 4 bytes (12.6 MB), more than the fixed scratch
    big = S.Workload(1, 16, 32, 6000, 64, causal=False, seed=25)
    dims = (big.B, big.H, big.n_q, big.n_k, big.d)
    Qb, Kb, Vb = (P.to_device(t) for t in S.make_qkv(big))
    ob = outputs(big)
    assert lamp.lamp_workspace_size(dims, lamp.LAMP_STRICT) > lamp.LAMP_NOALLOC_SCRATCH_BYTES
    rc = lamp.lamp_attention_noalloc(dims=dims, Q=Qb, K=Kb, V=Vb, out=ob["out"], mu=4, tau=0.1, check=False)
    assert rc == lamp.LAMP_ERR_WORKSPACE and "lamp_attention_ex" in lamp.lamp_last_error()

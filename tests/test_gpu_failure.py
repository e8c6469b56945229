"""The bounded-wait failure path of the whole-row kernel, on the GPU.

Every mbarrier wait in the kernels gives up after about two seconds of
%globaltimer, writes LAMP_ERR_TIMEOUT to the caller's status word and lets the
kernel end (after the tensor-core work in flight has drained and the tensor
memory is released), so that a protocol error never hangs the device. The
test-only field debug_stall = LAMP_DEBUG_STALL_PRODUCERS makes the score
producers hand over nothing, so that every other warp's wait runs out: nothing
traps, nothing waits without a limit. The test checks that the call ends by
itself, that the status word reads LAMP_ERR_TIMEOUT, and that a normal call
afterwards on the same context is still correct (against the oracle).
"""
import time

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


def test_wait_that_runs_out_reports_timeout_and_the_context_stays_usable():
    w = S.Workload(1, 2, 64, 64, 64, seed=31)  # rows short enough for the whole-row kernel
    Q, K, V = S.make_qkv(w)
    Qd, Kd, Vd = P.to_device(Q), P.to_device(K), P.to_device(V)
    dims = (w.B, w.H, w.n_q, w.n_k, w.d)
    out = torch.empty_like(Qd)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.time()
    lamp.lamp_attention_ex(dims=dims, Q=Qd, K=Kd, V=Vd, out=out, mu=4, tau=0.05, status_out=status,
                           debug_stall=lamp.LAMP_DEBUG_STALL_PRODUCERS)
    torch.cuda.synchronize()  # the kernel ends by itself
    elapsed = time.time() - t0
    assert status.item() == lamp.LAMP_ERR_TIMEOUT
    assert 1.0 < elapsed < 60.0, elapsed  # the waits gave up after their limit, not at once
    # the same context, normal calls: the status word stays clear and the results
    # match the oracle
    status2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    out2 = torch.empty_like(Qd)
    lamp.lamp_attention_ex(dims=dims, Q=Qd, K=Kd, V=Vd, out=out2, mu=4, tau=0.05, status_out=status2)
    g = P.GpuCall(w, Qd, Kd, Vd, mu=4, tau=0.05, variant=oracle.STRICT)
    assert status2.item() == 0
    assert torch.equal(out2, g.res.out)
    rows = np.arange(w.B * w.H * w.n_q, dtype=np.int64)
    orc = oracle.attention_rows(Q, K, V, causal=w.causal, mu=4, tau=0.05, variant=oracle.STRICT, rows=rows,
                                want_crit=True, threads=8)
    P.compare(w, g.rows(rows), orc, rows, 0.05, oracle.STRICT)

"""Benchmark of LAMP attention on B200: one JSON line on stdout (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--mu MU] [--rate R]

A step is one LAMP attention call over one batch of synthetic inputs: PS(mu)
scores, look-ahead selection, FP32 recompute of the selected scores, softmax
and P.V. The default workload is the GPT-2 XL attention shape (batch 1, 25
heads, 1024 causal tokens, d = 64), strict LAMP, mu = 4, tau from
tests/golden/tau.json for a 1.6 % recompute rate (computed by the oracle).

With N > 1 (torchrun, one process per GPU) every rank runs its own batch
(seed = rank): the (batch, head) units are independent, so there is no
collective on the data path and the scaling is weak. Timing: per step, CUDA
events around the call on the launching stream, L2 flushed (256 MB write)
between steps outside the events; the max over ranks is reported.

--impl reference times the CPU oracle (the plain C definition of the method)
on this host's cores on a bounded sample of the same workload.

The gelu_* and ln_* workloads time LAMP on an elementwise activation (GELU after
a PS(mu) linear map) and on LayerNorm after a PS(mu) linear map, with the same
contract.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as S  # noqa: E402

METRIC = "LAMP attention G-scores/s at 1x25x1024x64 mu=4; % of roofline; KL vs FP32"
UNIT = "G-scores/s"
TAU_FILE = os.path.join(ROOT, "tests", "golden", "tau.json")
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
L2_FLUSH_BYTES = 256 << 20
N_SM = 148
FP32_LANES_PER_SM_CLK = 128
VARIANT_NAMES = {0: "strict", 1: "relaxed", 2: "given_mask"}


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gpt2xl_1x25x1024x64", choices=sorted(S.WORKLOADS) + sorted(S.LINEAR_WORKLOADS))
    ap.add_argument("--variant", type=int, default=None, help="0 strict, 1 relaxed (default: per workload)")
    ap.add_argument("--mu", type=int, default=4)
    ap.add_argument("--rate", type=float, default=None, help="target recompute rate (tau from tau.json)")
    ap.add_argument("--no-kl", action="store_true", help="skip the accuracy evaluation")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffer) timing")
    return ap.parse_args()


DEFAULTS = {  # workload -> (variant, rate)
    "gpt2xl_1x25x1024x64": (0, 0.016),
    "batch8_8x25x1024x64": (1, 0.016),
    "long_1x32x16384x128": (1, 0.01),
    "long_1x8x4096x128": (1, 0.01),
    "decode_1x32x1x16384x128": (0, 0.016),
    "outlier_4x25x4096x64": (0, 0.003),
    "single_head_128": (0, None),
    "gelu_gpt2xl_fc_1024x6400x1600": (0, 0.016),
    "gelu_small_96x300x200": (0, 0.016),
    "ln_gpt2xl_proj_1024x1600x1600": (0, 0.016),
    "ln_small_64x300x128": (0, 0.016),
}


def lookup_tau(workload: str, variant: int, mu: int, rate: float | None) -> tuple[float, float | None]:
    """The calibrated tau as the binary32 value the C ABI receives (the value the
    GPU parity tests pass to both the kernels and the oracle)."""
    if workload == "single_head_128" and rate is None:
        return float(np.float32(0.05)), None
    doc = json.load(open(TAU_FILE))
    for e in doc["entries"]:
        if e["workload"] == workload and e["variant"] == variant and e["mu"] == mu and abs(e["rate"] - rate) < 1e-12:
            return float(np.float32(e["tau"])), float(e["rate"])
    raise SystemExit(f"no tau for {workload} variant={variant} mu={mu} rate={rate} in {TAU_FILE}")


def is_decode(w) -> bool:
    """The library's decode routing: few query rows per head against long rows."""
    return w.n_q <= 4 and w.n_k >= 512


def library_launches_per_call(w, variant: int) -> int:
    """The library's kernels in one attention call, by its routing: decode shapes run
    the scores and the selection kernels; the others the exponent-statistics kernel
    and one row kernel, and strict rows too long for the whole-row kernel (more than
    1024 keys at d = 64, 896 at d = 128) its two streamed passes."""
    if is_decode(w):
        return 2
    whole_row = w.n_k <= (1024 if w.d == 64 else 896)
    return 3 if (variant == 0 and not whole_row) else 2


def rank_workload(w, rank: int):
    """Weak scaling: every rank runs the same shape on its own inputs (seed + rank)."""
    return S.Workload(w.B, w.H, w.n_q, w.n_k, w.d, w.causal, w.outlier_frac, w.outlier_scale, seed=w.seed + rank)


def max_over_ranks(values, device):
    """Element-wise maximum of a few floats over all ranks (the step time of a job is
    its slowest rank's). Single process: the values themselves."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_value(world: int, valid_per_rank: int, ms: float) -> float:
    """Whole-job throughput in G-scores/s: every rank's scores over the slowest rank's time."""
    return world * valid_per_rank / (ms * 1e-3) / 1e9


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


# ----------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("timestamp,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None
        self.lines: list[str] = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        mhz, mx, reasons, n = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for (t, line) in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10 or (self.uuid and f[1] != self.uuid):
                continue
            if self.t0 and t < self.t0 - 0.05:
                continue
            if self.t1 and t > self.t1 + 0.25:
                continue
            n += 1
            try:
                mhz.append(float(f[2]))
                mx = float(f[3])
            except ValueError:
                continue
            for nm, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": n}


# ----------------------------------------------------------------------------------------
# reference arm: the CPU oracle on the host cores
# ----------------------------------------------------------------------------------------
def sample_rows_for(w: S.Workload, frac: float) -> np.ndarray:
    """Every m-th query row of every head (a bounded, evenly spread sample)."""
    total = w.B * w.H * w.n_q
    m = max(1, int(round(1.0 / frac)))
    return np.arange(0, total, m, dtype=np.int64)


def valid_in_rows(w: S.Workload, rows: np.ndarray) -> int:
    return int(sum(w.valid_keys(int(r) % w.n_q) for r in rows))


def oracle_rate(w, Q, K, V, mu, tau, variant, rows, threads) -> tuple[float, float]:
    import oracle
    t0 = time.perf_counter()
    oracle.attention_rows(Q, K, V, causal=w.causal, mu=mu, tau=tau, variant=variant, rows=rows,
                          want_scores=False, threads=threads)
    dt = time.perf_counter() - t0
    return valid_in_rows(w, rows) / dt / 1e9, dt


def run_reference(a, w, variant, mu, tau, cfg):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    threads = os.cpu_count() or 1
    Q, K, V = S.make_qkv(w)
    # each step: a fixed sample of rows sized to about 0.1-0.5 s on the host's cores
    frac = min(1.0, 2.0e6 / max(1, w.valid_scores()))
    rows = sample_rows_for(w, frac)
    for _ in range(a.warmup):
        oracle_rate(w, Q, K, V, mu, tau, variant, rows, threads)
    times = []
    for _ in range(a.steps):
        _, dt = oracle_rate(w, Q, K, V, mu, tau, variant, rows, threads)
        times.append(dt)
    per = valid_in_rows(w, rows)
    ms = 1e3 * statistics.mean(times)
    value = per / (ms * 1e-3) / 1e9
    sample = f"{rows.size} of {w.B * w.H * w.n_q} query rows (every {int(round(1 / frac))}th), {per} scores per step"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": cfg, "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------------------
def source_hash(files) -> str:
    """Hash of the named csrc files: a traffic figure is valid only for the sources it
    was measured on."""
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "mixed_precision_attention_ps_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def traffic_bytes(workload: str, variant: int, mu: int) -> float | None:
    """DRAM bytes per launch of the measured kernel from the committed ncu summary,
    or None when that kernel's sources changed since the capture."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    doc = json.load(open(TRAFFIC_FILE))
    for e in doc.get("entries", []):
        if e["workload"] == workload and e["variant"] == variant and e["mu"] == mu:
            if source_hash(e["sources"]) != e["source_hash"]:
                return None
            return float(e["dram_bytes_per_launch"])
    return None


def kl_eval(lamp, torch, w, Qd, Kd, Vd, mu, tau, variant, stream):
    """Mean row KL(P_fp32 || P_x) for no recompute, LAMP at tau, and a random
    selection of the same per-row count (evaluation only, outside the timed region)."""
    def run(**kw):
        r = lamp.attention(Qd, Kd, Vd, mu=mu, causal=w.causal, want_scores=True, want_count=True, stream=stream, **kw)
        torch.cuda.synchronize()
        return r

    def mean_kl(ref, x):
        lp = torch.log_softmax(ref.double(), dim=-1)
        lq = torch.log_softmax(x.double(), dim=-1)
        p = lp.exp()
        t = torch.where(p > 0, p * (lp - lq), torch.zeros_like(p))
        kl = t.sum(-1)
        valid = torch.isfinite(ref).any(-1)
        return float(kl[valid].mean().item())

    ref = run(tau=-1.0, variant=0).mixed_scores
    base = run(tau=float("inf"), variant=0).mixed_scores
    lr = run(tau=tau, variant=variant)
    kl0 = mean_kl(ref, base)
    kl_l = mean_kl(ref, lr.mixed_scores)
    counts = lr.mask.view(torch.int32).cpu().numpy().view(np.uint32)
    per_row = np.unpackbits(counts.view(np.uint8), axis=-1).sum(-1).reshape(w.B * w.H, w.n_q)
    rmask = S.random_control_mask(w, per_row).reshape(w.B, w.H, w.n_q, -1)
    rr = run(tau=0.0, variant=2, mask_in=torch.from_numpy(rmask.view(np.int32)).cuda())
    kl_r = mean_kl(ref, rr.mixed_scores)
    rate = lr.n_selected.item() / w.valid_scores()
    return {"recompute_rate": rate, "kl_ps_only": kl0, "kl_lamp": kl_l, "kl_random_same_count": kl_r,
            "kl_reduction_lamp": kl0 / kl_l if kl_l > 0 else None,
            "kl_reduction_random": kl0 / kl_r if kl_r > 0 else None,
            "pages_mu4_context": "GPT-2 XL model-output KL reductions 12x @0.3%, 83x @1.6%, 385x @7.6% "
                                 "(simulation; a different quantity)"}


def run_ours(a, w, variant, mu, tau, cfg):
    import torch
    import torch.distributed as dist

    import mixed_precision_attention_ps_b200 as lamp

    rank, local, world = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    lamp.load()
    wr = rank_workload(w, rank)
    Q, K, V = S.make_qkv(wr)

    def dev_t(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(dev).view(torch.bfloat16)

    Qd, Kd, Vd = dev_t(Q), dev_t(K), dev_t(V)
    dims = (w.B, w.H, w.n_q, w.n_k, w.d)
    nwords = (w.n_k + 31) // 32
    out = torch.empty_like(Qd)
    mask = torch.empty((w.B, w.H, w.n_q, nwords), dtype=torch.int32, device=dev)
    ws_bytes = lamp.lamp_workspace_size(dims, variant)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    args = lamp.make_args(dims, Qd, Kd, Vd, out, mask_out=mask, mu=mu, tau=tau, variant=variant,
                          causal=int(w.causal), stream=stream, workspace=ws, workspace_bytes=ws_bytes)
    call = lambda: lamp.lamp_attention_ex(args)  # noqa: E731
    valid = wr.valid_scores()

    # ---- device-resident timing --------------------------------------------------------
    props = torch.cuda.get_device_properties(dev)
    clocks = ClockSampler(getattr(props, "uuid", None) and ("GPU-" + str(props.uuid)))
    clocks.start()
    for _ in range(a.warmup):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark("t0")
    for s, e in evs:
        flush.zero_()
        s.record(stream)
        call()
        e.record(stream)
    torch.cuda.synchronize()
    clocks.mark("t1")
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    times = [s.elapsed_time(e) for s, e in evs]
    ms = max_over_ranks([statistics.mean(times)], dev)[0]
    launches_per_step = library_launches_per_call(w, variant)

    # ---- end to end through the C ABI with host buffers ---------------------------------
    # Every step copies its inputs from pinned host memory and reads its output and
    # mask back, inside the timed region. Two forms are measured:
    #   serial:    H2D, call and D2H of a step one after another on one stream;
    #   pipelined: two device buffer sets and three streams (H2D, compute, D2H), so
    #              step i's copies overlap step i - 1's call, as a serving loop would
    #              run; ordering by events (the call waits for its inputs, a buffer
    #              set is refilled only after its output has been read back).
    # e2e.value is the pipelined throughput over all steps (first H2D to last D2H).
    hQ, hK, hV = (torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).pin_memory() for x in (Q, K, V))
    hout = [torch.empty(out.shape, dtype=torch.int16).pin_memory() for _ in range(2)]
    hmask = [torch.empty(mask.shape, dtype=torch.int32).pin_memory() for _ in range(2)]
    e2e_steps = 0 if a.no_e2e else max(3, min(a.steps, 500))
    ms_serial = ms_e2e = float("nan")
    if e2e_steps:
        Qi, Ki, Vi = Qd.view(torch.int16), Kd.view(torch.int16), Vd.view(torch.int16)
        for _ in range(3):
            Qi.copy_(hQ, non_blocking=True); Ki.copy_(hK, non_blocking=True); Vi.copy_(hV, non_blocking=True)
            call()
            hout[0].copy_(out.view(torch.int16), non_blocking=True); hmask[0].copy_(mask, non_blocking=True)
        torch.cuda.synchronize()
        evs2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
        for s, e in evs2:
            s.record(stream)
            Qi.copy_(hQ, non_blocking=True); Ki.copy_(hK, non_blocking=True); Vi.copy_(hV, non_blocking=True)
            call()
            hout[0].copy_(out.view(torch.int16), non_blocking=True); hmask[0].copy_(mask, non_blocking=True)
            e.record(stream)
        torch.cuda.synchronize()
        ms_serial = statistics.mean(s.elapsed_time(e) for s, e in evs2)

        # pipelined
        sets = []
        for b in range(2):
            bq, bk, bv = (torch.empty_like(x) for x in (Qd, Kd, Vd))
            bo, bm = torch.empty_like(out), torch.empty_like(mask)
            bws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
            sets.append((bq, bk, bv, bo, bm, bws))
        s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        bargs = [lamp.make_args(dims, st[0], st[1], st[2], st[3], mask_out=st[4], mu=mu, tau=tau, variant=variant,
                                causal=int(w.causal), stream=s_cmp, workspace=st[5], workspace_bytes=ws_bytes)
                 for st in sets]

        def pipeline(n):
            done_in = [torch.cuda.Event() for _ in range(n)]
            done_cmp = [torch.cuda.Event() for _ in range(n)]
            done_out = [torch.cuda.Event() for _ in range(n)]
            for i in range(n):
                b = i & 1
                bq, bk, bv, bo, bm, _ = sets[b]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(done_cmp[i - 2])  # the call that read this set is done
                    bq.view(torch.int16).copy_(hQ, non_blocking=True)
                    bk.view(torch.int16).copy_(hK, non_blocking=True)
                    bv.view(torch.int16).copy_(hV, non_blocking=True)
                    done_in[i].record(s_in)
                s_cmp.wait_event(done_in[i])
                if i >= 2:
                    s_cmp.wait_event(done_out[i - 2])  # this set's output has been read back
                lamp.lamp_attention_ex(bargs[b])
                done_cmp[i].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(done_cmp[i])
                    hout[b].copy_(bo.view(torch.int16), non_blocking=True)
                    hmask[b].copy_(bm, non_blocking=True)
                    done_out[i].record(s_out)
            return done_out[n - 1]

        pipeline(4)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(s_in)
        last = pipeline(e2e_steps)
        s_out.wait_event(last)
        t1.record(s_out)
        torch.cuda.synchronize()
        ms_e2e = t0.elapsed_time(t1) / e2e_steps
        # the pipelined outputs equal the device-resident call's
        assert torch.equal(hout[(e2e_steps - 1) & 1], out.view(torch.int16).cpu())
    ms_e2e, ms_serial = max_over_ranks([ms_e2e, ms_serial], dev)
    if world > 1:
        dist.barrier()
    h2d = Q.nbytes + K.nbytes + V.nbytes
    d2h = out.numel() * 2 + mask.numel() * 4

    result = None
    if rank == 0:
        value = job_value(world, valid, ms)
        value_e2e = job_value(world, valid, ms_e2e)
        # roofline: ALU issue. 4 d lane-ops per valid score (1 multiply-add + 3 integer
        # ops of the round-to-nearest-even to mu bits, per accumulation step), against
        # 128 FP32/INT32 lanes per SM per clock x 148 SMs x the maximum SM clock.
        peaks = json.load(open(PEAKS_FILE)) if os.path.exists(PEAKS_FILE) else {}
        f_max = float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
        peak = N_SM * FP32_LANES_PER_SM_CLK * f_max / 1e12
        achieved = 4.0 * w.d * valid / (ms * 1e-3) / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Tlane-op/s",
                "frac": achieved / peak, "traffic": traffic_bytes(a.workload, variant, mu),
                "kernel": "one call: exponent-statistics kernel + the row kernel for the shape "
                          "(ws_kernel for n_k <= 1024 at d = 64); the row kernel is ~97% of the call",
                "peak_basis": f"148 SMs x 128 lanes/clk x {f_max / 1e6:.0f} MHz (max SM clock)"}
        if is_decode(w):
            # decode shapes stream K and V once per call: HBM bounds them. Algorithmic
            # bytes: K and V read, Q read, out and mask written (the score scratch is
            # L2 resident).
            nbytes = (2 * w.B * w.H * w.n_k * w.d * 2 + 2 * w.B * w.H * w.n_q * w.d * 2
                      + w.B * w.H * w.n_q * ((w.n_k + 31) // 32) * 4)
            hbm = float(peaks.get("hbm_gbs", 6650.0))
            gbs = nbytes / (ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                    "traffic": traffic_bytes(a.workload, variant, mu), "bytes_per_call": nbytes,
                    "kernel": "one call: exponent statistics + the three decode kernels (scores and chunk "
                              "statistics, selection and partial P.V, combine)",
                    "peak_basis": "MEASURED_PEAKS.json hbm_gbs (copy)" if "hbm_gbs" in peaks
                                  else "fallback 6650 GB/s",
                    "alu_frac": achieved / peak}
        result = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
                  "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                  "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": cfg,
                  "clocks": clk, "roofline": roof, "gpu_launches": launches_per_step * a.steps,
                  "e2e": {"value": value_e2e, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                          "ms_per_step": ms_e2e, "form": "pipelined: 2 buffer sets, H2D / compute / D2H streams",
                          "ms_per_step_serial": ms_serial,
                          "value_serial": world * valid / (ms_serial * 1e-3) / 1e9 if ms_serial == ms_serial else None},
                  "attention_gflops": 4.0 * w.d * valid / (ms * 1e-3) / 1e9 * world,
                  "ms_p10_p90": [float(np.percentile(times, 10)), float(np.percentile(times, 90))]}
    # accuracy evaluation (rank 0, outside the timed region)
    if rank == 0 and not a.no_kl:
        result["accuracy"] = kl_eval(lamp, torch, wr, Qd, Kd, Vd, mu, tau, variant, stream)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if not a.no_cpu_baseline and world == 1:
            result["cpu_baseline"] = cpu_baseline(wr, Q, K, V, mu, tau, variant)
        print(json.dumps(result), flush=True)
    return 0


def cpu_baseline(w, Q, K, V, mu, tau, variant) -> dict:
    """The oracle as it stands, on the host's cores, over whole-workload passes
    (or row samples of it) until about 10 s of work have run."""
    threads = os.cpu_count() or 1
    total = w.valid_scores()
    frac = min(1.0, 1.5e8 / total)
    rows = sample_rows_for(w, frac)
    per = valid_in_rows(w, rows)
    t_all, n_scores, passes = 0.0, 0, 0
    while t_all < 10.0 and passes < 20:
        _, dt = oracle_rate(w, Q, K, V, mu, tau, variant, rows, threads)
        t_all += dt
        n_scores += per
        passes += 1
    sample = (f"{passes} pass(es) over {rows.size} of {w.B * w.H * w.n_q} query rows"
              f" ({per} scores each), {t_all:.1f} s")
    return {"value": n_scores / t_all / 1e9, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample}


# ----------------------------------------------------------------------------------------
# LAMP on the operators after a PS(mu) linear map: GELU(scale * x W^T) (op "gelu")
# and LayerNorm(scale * x W^T) (op "ln")
# ----------------------------------------------------------------------------------------
def linear_metric(lw, mu, op="gelu") -> str:
    name = "LayerNorm" if op == "ln" else "GELU"
    return f"LAMP {name}(x W^T) G-outputs/s at {lw.M}x{lw.N}x{lw.K} mu={mu}; % of roofline"


LINEAR_UNIT = "G-outputs/s"


def linear_map_launches(M: int, N: int, num_sms: int) -> int:
    """Kernel launches of the library's linear map for an M x N output (its tile-width
    rule: 64-wide tiles for the whole problem, or 128-wide tiles in whole rounds of
    2 x num_sms CTAs plus a second launch of 64-wide tiles for a last partial round)."""
    rt = (M + 63) // 64
    c4, c2 = (N + 127) // 128, (N + 63) // 64
    t4, t2 = rt * c4, rt * c2
    share4, share2 = (t4 + num_sms - 1) // num_sms * 2, (t2 + num_sms - 1) // num_sms
    if 8 * share2 <= 7 * share4:
        return 1
    full = t4 // (2 * num_sms) * (2 * num_sms)
    return 2 if (full > 0 and 0 < t4 - full < 2 * num_sms and c2 == 2 * c4) else 1


def linear_oracle_pass(lw, x, W, mu, tau, rows, threads, op="gelu") -> float:
    import oracle
    t0 = time.perf_counter()
    if op == "ln":
        oracle.linear_ln_rows(x, W, scale=lw.scale, mu=mu, tau=tau, rows=rows, threads=threads)
    else:
        oracle.linear_gelu_rows(x, W, scale=lw.scale, mu=mu, tau=tau, rows=rows, threads=threads)
    return time.perf_counter() - t0


def linear_cpu_baseline(lw, x, W, mu, tau, seconds=10.0, op="gelu") -> dict:
    """The activation oracle as it stands, on the host's cores, over a row sample
    repeated until about `seconds` of work have run."""
    threads = os.cpu_count() or 1
    m = max(1, lw.M // max(1, int(1.5e8 // (lw.N * lw.K))))
    rows = np.arange(0, lw.M, m, dtype=np.int64)
    t_all, n_out, passes = 0.0, 0, 0
    while t_all < seconds and passes < 20:
        t_all += linear_oracle_pass(lw, x, W, mu, tau, rows, threads, op)
        n_out += rows.size * lw.N
        passes += 1
    return {"value": n_out / t_all / 1e9, "unit": LINEAR_UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{passes} pass(es) over {rows.size} of {lw.M} rows (every {m}th, {rows.size * lw.N} "
                      f"outputs each), {t_all:.1f} s"}


def linear_accuracy(lamp, torch, lw, xd, Wd, mu, tau, stream, op="gelu") -> dict:
    """Errors against the all-FP32 outputs (tau < 0) for no recompute, LAMP at tau and
    a random choice of the same per-row count, on a row sample (outside the timed region)."""
    import oracle

    fn = lamp.linear_layernorm if op == "ln" else lamp.linear_gelu

    def run(**kw):
        r = fn(xd, Wd, mu=mu, scale=lw.scale, want_scores=True, want_out_f32=True, want_count=True, stream=stream,
               **kw)
        torch.cuda.synchronize()
        return r

    rows = torch.arange(0, lw.M, 8, device=xd.device)
    pick = lambda t: t.index_select(0, rows).cpu().numpy()  # noqa: E731
    ref = run(tau=-1.0)
    base = run(tau=float("inf"))
    lr = run(tau=tau)
    words = lr.mask.cpu().numpy().view(np.uint32)
    per_row = np.unpackbits(words.view(np.uint8), axis=-1).sum(-1)
    rmask = S.linear_random_mask(lw, per_row)
    rr = run(tau=0.0, variant=2, mask_in=torch.from_numpy(rmask.view(np.int32)).to(xd.device))
    r_out, r_y = pick(ref.out_f32), pick(ref.mixed)
    cases = (("ps_only", base), ("lamp", lr), ("random_same_count", rr))
    if op == "ln":
        err = {k: oracle.ln_errors(pick(v.out_f32), r_out) for k, v in cases}
        key = "mean_l2"
    else:
        err = {k: oracle.act_errors(pick(v.out_f32), pick(v.mixed), r_out, r_y) for k, v in cases}
        key = "max_amp"
    return {"recompute_rate": lr.n_selected.item() / lw.outputs(), "rows_sampled": int(rows.numel()),
            "errors_vs_fp32": err,
            f"{key}_reduction_lamp": err["ps_only"][key] / max(err["lamp"][key], 1e-300),
            f"{key}_reduction_random": err["ps_only"][key] / max(err["random_same_count"][key], 1e-300)}


def run_linear_reference(a, lw, mu, tau, cfg, op="gelu"):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    threads = os.cpu_count() or 1
    x, W = S.make_linear(lw)
    m = max(1, lw.M // max(1, int(1.6e8 // (lw.N * lw.K))))
    rows = np.arange(0, lw.M, m, dtype=np.int64)
    for _ in range(a.warmup):
        linear_oracle_pass(lw, x, W, mu, tau, rows, threads, op)
    times = [linear_oracle_pass(lw, x, W, mu, tau, rows, threads, op) for _ in range(a.steps)]
    ms = 1e3 * statistics.mean(times)
    value = rows.size * lw.N / (ms * 1e-3) / 1e9
    sample = f"{rows.size} of {lw.M} rows (every {m}th), {rows.size * lw.N} outputs per step"
    line = {"metric": linear_metric(lw, mu, op), "value": value, "unit": LINEAR_UNIT, "n_gpus": a.gpus, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": cfg, "impl": "reference",
            "cpu_baseline": {"value": value, "unit": LINEAR_UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": LINEAR_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_linear_ours(a, lw, mu, tau, cfg, op="gelu"):
    import torch
    import torch.distributed as dist

    import mixed_precision_attention_ps_b200 as lamp

    rank, local, world = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    lamp.load()
    lwr = S.LinearWorkload(lw.M, lw.N, lw.K, seed=lw.seed + rank)  # weak scaling: own inputs per rank
    x, W = S.make_linear(lwr)

    def dev_t(v):
        return torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).to(dev).view(torch.bfloat16)

    xd, Wd = dev_t(x), dev_t(W)
    out = torch.empty((lw.M, lw.N), dtype=torch.bfloat16, device=dev)
    mask = torch.empty((lw.M, (lw.N + 31) // 32), dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    ws_bytes = lamp.lamp_ln_workspace_size(lw.M, lw.N) if op == "ln" else 0

    def make(x_, W_, out_, mask_, st_):
        if op == "ln":  # the LayerNorm op's y_hat scratch comes from the caller here
            wsb = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
            return (lamp.make_ln_args(lw.M, lw.N, lw.K, x_, W_, out_, mask_out=mask_, mu=mu, tau=tau,
                                      scale=lw.scale, workspace=wsb, workspace_bytes=ws_bytes, stream=st_), wsb)
        return lamp.make_gelu_args(lw.M, lw.N, lw.K, x_, W_, out_, mask_out=mask_, mu=mu, tau=tau, scale=lw.scale,
                                   stream=st_), None

    entry = lamp.lamp_linear_layernorm if op == "ln" else lamp.lamp_linear_gelu
    args, keep = make(xd, Wd, out, mask, stream)
    call = lambda: entry(args)  # noqa: E731

    props = torch.cuda.get_device_properties(dev)
    clocks = ClockSampler(getattr(props, "uuid", None) and ("GPU-" + str(props.uuid)))
    clocks.start()
    for _ in range(a.warmup):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark("t0")
    for s, e in evs:
        flush.zero_()
        s.record(stream)
        call()
        e.record(stream)
    torch.cuda.synchronize()
    clocks.mark("t1")
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    times = [s.elapsed_time(e) for s, e in evs]
    ms = max_over_ranks([statistics.mean(times)], dev)[0]

    # end to end through the C ABI with host buffers, pipelined as for attention: two
    # device buffer sets, H2D / compute / D2H streams ordered by events
    hx, hW = (torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).pin_memory() for v in (x, W))
    hout = [torch.empty(out.shape, dtype=torch.int16).pin_memory() for _ in range(2)]
    hmask = [torch.empty(mask.shape, dtype=torch.int32).pin_memory() for _ in range(2)]
    e2e_steps = 0 if a.no_e2e else max(3, min(a.steps, 200))
    ms_e2e = float("nan")
    if e2e_steps:
        sets = [(torch.empty_like(xd), torch.empty_like(Wd), torch.empty_like(out), torch.empty_like(mask))
                for _ in range(2)]
        s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        bargs = [make(st[0], st[1], st[2], st[3], s_cmp) for st in sets]

        def pipeline(n):
            done_in = [torch.cuda.Event() for _ in range(n)]
            done_cmp = [torch.cuda.Event() for _ in range(n)]
            done_out = [torch.cuda.Event() for _ in range(n)]
            for i in range(n):
                b = i & 1
                bx, bW, bo, bm = sets[b]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(done_cmp[i - 2])
                    bx.view(torch.int16).copy_(hx, non_blocking=True)
                    bW.view(torch.int16).copy_(hW, non_blocking=True)
                    done_in[i].record(s_in)
                s_cmp.wait_event(done_in[i])
                if i >= 2:
                    s_cmp.wait_event(done_out[i - 2])
                entry(bargs[b][0])
                done_cmp[i].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(done_cmp[i])
                    hout[b].copy_(bo.view(torch.int16), non_blocking=True)
                    hmask[b].copy_(bm, non_blocking=True)
                    done_out[i].record(s_out)
            return done_out[n - 1]

        pipeline(4)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(s_in)
        last = pipeline(e2e_steps)
        s_out.wait_event(last)
        t1.record(s_out)
        torch.cuda.synchronize()
        ms_e2e = t0.elapsed_time(t1) / e2e_steps
        assert torch.equal(hout[(e2e_steps - 1) & 1], out.view(torch.int16).cpu())
    ms_e2e = max_over_ranks([ms_e2e], dev)[0]
    if world > 1:
        dist.barrier()
    result = None
    if rank == 0:
        n_out = lw.outputs()
        value = job_value(world, n_out, ms)
        peaks = json.load(open(PEAKS_FILE)) if os.path.exists(PEAKS_FILE) else {}
        f_max = float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
        peak = N_SM * FP32_LANES_PER_SM_CLK * f_max / 1e12
        achieved = 4.0 * lw.K * n_out / (ms * 1e-3) / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Tlane-op/s", "frac": achieved / peak,
                "traffic": traffic_bytes(a.workload, 0, mu),
                "kernel": ("one call: the linear-map kernel (gelu_kernel, store epilogue) + ln_rows_kernel"
                           if op == "ln" else "one call: gelu_kernel (128-wide tiles, then 64-wide tiles "
                                              "for a last partial round)"),
                "peak_basis": f"148 SMs x 128 lanes/clk x {f_max / 1e6:.0f} MHz (max SM clock); 4 K lane-ops "
                              "per output (K steps of 1 multiply-add + 3 integer ops of the rounding)"}
        result = {"metric": linear_metric(lw, mu, op), "value": value, "unit": LINEAR_UNIT, "n_gpus": world, "steps": a.steps,
                  "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                  "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": cfg, "clocks": clk,
                  "roofline": roof,
                  "gpu_launches": (linear_map_launches(lw.M, lw.N, props.multi_processor_count)
                                   + (1 if op == "ln" else 0)) * a.steps,
                  "e2e": {"value": job_value(world, n_out, ms_e2e), "unit": LINEAR_UNIT,
                          "h2d_bytes_per_step": x.nbytes + W.nbytes,
                          "d2h_bytes_per_step": out.numel() * 2 + mask.numel() * 4, "ms_per_step": ms_e2e,
                          "form": "pipelined: 2 buffer sets, H2D / compute / D2H streams"},
                  "ms_p10_p90": [float(np.percentile(times, 10)), float(np.percentile(times, 90))]}
        if not a.no_kl:
            result["accuracy"] = linear_accuracy(lamp, torch, lwr, xd, Wd, mu, tau, stream, op)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if not a.no_cpu_baseline and world == 1:
            result["cpu_baseline"] = linear_cpu_baseline(lwr, x, W, mu, tau, op=op)
        print(json.dumps(result), flush=True)
    return 0


def main_linear(a):
    lw = S.LINEAR_WORKLOADS[a.workload]
    op = "ln" if a.workload.startswith("ln_") else "gelu"
    _, drate = DEFAULTS[a.workload]
    rate = drate if a.rate is None else a.rate
    tau, rate = lookup_tau(a.workload, 0, a.mu, rate)
    cfg = {"workload": a.workload, "M": lw.M, "N": lw.N, "K": lw.K,
           "op": ("LayerNorm (no affine, eps = 1e-5) of scale * x W^T, greedy by sorted magnitude" if op == "ln"
                  else "GELU (tanh form) of scale * x W^T, kappa test"),
           "scale": lw.scale, "mu": a.mu, "tau": tau, "target_recompute_rate": rate,
           "inputs": "bf16 N(0,1) x and W (SplitMix64 + Box-Muller), seed = rank",
           "l2": "flushed between steps (256 MB write)", "outputs_per_step_per_gpu": lw.outputs()}
    if a.impl == "reference":
        return run_linear_reference(a, lw, a.mu, tau, cfg, op)
    return run_linear_ours(a, lw, a.mu, tau, cfg, op)


def main():
    a = parse()
    if a.workload in S.LINEAR_WORKLOADS:
        return main_linear(a)
    w = S.WORKLOADS[a.workload]
    dv, drate = DEFAULTS[a.workload]
    variant = dv if a.variant is None else a.variant
    rate = drate if a.rate is None else a.rate
    tau, rate = lookup_tau(a.workload, variant, a.mu, rate)
    cfg = {"workload": a.workload, "B": w.B, "H": w.H, "n_q": w.n_q, "n_k": w.n_k, "d": w.d, "causal": w.causal,
           "variant": VARIANT_NAMES[variant], "mu": a.mu, "tau": tau, "target_recompute_rate": rate,
           "inputs": "bf16 N(0,1) (SplitMix64 + Box-Muller), seed = rank", "l2": "flushed between steps (256 MB write)",
           "valid_scores_per_step_per_gpu": w.valid_scores()}
    if a.impl == "reference":
        return run_reference(a, w, variant, a.mu, tau, cfg)
    return run_ours(a, w, variant, a.mu, tau, cfg)


if __name__ == "__main__":
    sys.exit(main())

"""The multi-process side of bench.py on the CPU: two ranks over gloo.

The path shards with no exchange step (every rank runs its own batch, seeded by
its rank); the only collectives are the barrier and the maximum of the step
times over the ranks, from which the whole-job throughput is computed. These
tests run that logic with world size 2 over gloo (no GPU), and the reference
arm under torchrun, where rank 0 alone runs and prints.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench
    import synthetic as S

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # each rank's step times differ; the job takes the slowest rank's
        mx = bench.max_over_ranks([1.0 + rank, 10.0 - 3.0 * rank], torch.device("cpu"))
        w = bench.rank_workload(S.WORKLOADS["single_head_128"], rank)
        seed_first_q = int(S.make_qkv(w)[0].reshape(-1)[0])
        dist.barrier()
        out.put((rank, mx, w.seed, seed_first_q, bench.job_value(world, w.valid_scores(), mx[0])))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo():
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(world))
    for rank, mx, seed, _, value in res:
        assert mx == [2.0, 10.0]  # element-wise maximum over the two ranks
        assert seed == rank       # weak scaling: the rank's own inputs
        # 2 ranks x 8256 scores (the single-head workload) in 2 ms
        assert value == pytest.approx(2 * 8256 / 2e-3 / 1e9)
    assert res[0][3] != res[1][3]  # different inputs on the two ranks


def test_single_process_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([3.5, 1.25], None) == [3.5, 1.25]
    assert bench.job_value(1, 1000, 1.0) == pytest.approx(1e-3)


def test_reference_arm_under_torchrun_prints_once():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "single_head_128"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"


@pytest.mark.parametrize("workload", ["gelu_small_96x300x200", "ln_small_64x300x128"])
def test_operator_reference_arms_under_torchrun(workload):
    """The activation and LayerNorm workloads' reference arms (the oracle) under
    torchrun: rank 0 alone runs and prints one line with the contract's keys."""
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", workload]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "G-outputs/s" and d["value"] > 0
    assert d["config"]["workload"] == workload and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle"


def test_linear_map_launch_count_follows_the_tile_rule():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.linear_map_launches(1024, 6400, 148) == 2   # 592 wide tiles, then 416 narrow ones
    assert bench.linear_map_launches(1024, 1600, 148) == 1   # narrow tiles for the whole problem
    assert bench.linear_map_launches(96, 300, 148) == 1
    assert bench.linear_map_launches(1024, 6304, 148) == 1  # 50 wide but 99 narrow column tiles: no split


def test_every_bench_default_has_a_calibrated_tau():
    """bench.py's default (workload, variant, rate) pairs all resolve in tau.json,
    so no GPU run stops on a missing threshold."""
    sys.path.insert(0, ROOT)
    import bench
    import synthetic as S

    for name, (variant, rate) in bench.DEFAULTS.items():
        assert name in S.WORKLOADS or name in S.LINEAR_WORKLOADS
        tau, r = bench.lookup_tau(name, variant, 4, rate)
        assert tau == tau and (rate is None or r == rate)

"""Host-side logic of bench.py that its JSON line depends on (no GPU needed):
the calibrated tau it passes across the C ABI, the launch count it claims per
call, and the traffic figure it reads from the committed ncu summaries."""
import json

import numpy as np

import bench
import synthetic as S


def test_tau_is_the_binary32_value_of_the_stored_threshold():
    doc = json.load(open(bench.TAU_FILE))
    e = next(e for e in doc["entries"] if e["workload"] == "gpt2xl_1x25x1024x64" and e["mu"] == 4)
    tau, rate = bench.lookup_tau(e["workload"], e["variant"], e["mu"], e["rate"])
    assert tau == float(np.float32(e["tau"]))
    assert rate == e["rate"]


def test_launch_count_follows_the_kernel_routing():
    W = S.WORKLOADS
    # whole-row kernel: statistics + one row kernel, any variant
    assert bench.library_launches_per_call(W["gpt2xl_1x25x1024x64"], 0) == 2
    assert bench.library_launches_per_call(W["batch8_8x25x1024x64"], 1) == 2
    # rows past the whole-row kernel: one streamed pass for relaxed, two for strict
    assert bench.library_launches_per_call(W["long_1x32x16384x128"], 1) == 2
    assert bench.library_launches_per_call(W["outlier_4x25x4096x64"], 0) == 3
    assert bench.library_launches_per_call(S.Workload(1, 2, 900, 900, 128), 0) == 3
    assert bench.library_launches_per_call(S.Workload(1, 2, 896, 896, 128), 0) == 2
    # decode: the scores and the selection kernels, no statistics pass
    assert bench.library_launches_per_call(W["decode_1x32x1x16384x128"], 0) == 2
    assert bench.library_launches_per_call(W["decode_1x32x1x16384x128"], 1) == 2


def test_traffic_figure_holds_only_for_the_sources_it_was_measured_on(tmp_path, monkeypatch):
    doc = json.load(open(bench.TRAFFIC_FILE))
    for e in doc["entries"]:  # the committed figures match the committed sources
        assert bench.traffic_bytes(e["workload"], e["variant"], e["mu"]) == float(e["dram_bytes_per_launch"])
    stale = json.loads(json.dumps(doc))
    stale["entries"][0]["source_hash"] = "0" * 16
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(stale))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    e0 = stale["entries"][0]
    assert bench.traffic_bytes(e0["workload"], e0["variant"], e0["mu"]) is None
    assert bench.traffic_bytes("no_such_workload", 0, 4) is None

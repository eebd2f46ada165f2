"""Host-side logic of bench.py that needs no GPU."""
import os
import sys

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))
import bench  # noqa: E402


def test_traffic_key_ignores_comments_but_not_code():
    """The DRAM-traffic record is keyed to the code of the sources that decide
    the GEMM launch mix: editing a comment keeps the key, editing code (even a
    constant) changes it, so a stale capture is reported as null."""
    src = "int f(int a) {  // scale\n  /* block\n comment */ return 2 * a;\n}\n"
    same = "int f(int a) {   // a different comment\n\n  return 2 * a;   \n}\n"
    other = "int f(int a) {\n  return 3 * a;\n}\n"
    key = lambda text: bench.traffic_source_sha(lambda name: text)
    assert key(src) == key(same)
    assert key(src) != key(other)


def test_traffic_record_is_well_formed():
    """The committed record names its capture, workload and solver, and
    carries a positive per-launch byte count with the key it was taken on."""
    import json
    with open(os.path.join(bench.ROOT, "profiles", "gemm_traffic.json")) as f:
        d = json.load(f)
    assert d["bytes_per_launch"] > 0 and d["captured_launches"] > 0
    assert d["workload_key"] in bench.WORKLOAD_NAMES.values() or d["workload_key"].startswith("llama_1b_shapes")
    assert d["solver"] in bench.SOLVER_NAMES.values()
    assert len(d["source_sha256"]) == 64 and "ncu" in d["command"]


def test_cpu_baseline_reports_a_single_thread_number():
    """The oracle baseline of the default workload carries, beside the
    multi-threaded rate, a one-thread rate on a bounded sample."""
    import workloads
    out = bench.cpu_baseline(workloads.workload("lowrank"), 2.0)
    assert out["kind"] == "oracle" and out["value"] > 0 and out["cores"] >= 1
    one = out.get("single_thread")
    assert one is not None and one["cores"] == 1 and one["value"] > 0
    assert "1 thread" in one["sample"]


def test_step_time_split_by_refresh():
    """A 20-step window starting on a refresh, refresh every 10: steps 0 and
    10 are the refresh steps; every step counts once."""
    ms = [5.0 if k % 10 == 0 else 0.2 for k in range(20)]
    out = bench.split_step_ms(ms, 10)
    assert out["refresh_steps"] == 2 and out["non_refresh_steps"] == 18
    assert out["refresh_ms"] == 5.0 and abs(out["non_refresh_ms"] - 0.2) < 1e-12
    every_step = bench.split_step_ms([3.0, 4.0], 1)       # refresh every step
    assert every_step["refresh_ms"] == 3.5 and every_step["non_refresh_ms"] is None
    assert bench.refresh_steps(20, 10) == out["refresh_steps"]


def test_workload_label_marks_a_cut_llama_workload():
    """--layers cuts the Llama workload for small profiling captures; its label
    (and so the traffic record's key) must not be the full workload's."""
    import workloads
    full = workloads.workload("llama")
    cut = workloads.workload("llama", shapes=full.shapes[:bench.LLAMA_LAYER * 2])
    assert bench.workload_label(full) == "llama_1b_shapes_b1024"
    assert bench.workload_label(cut) == "llama_1b_shapes_b1024_2layers"

"""Host logic of bench.py that needs no GPU: the traffic counters are used
only on the sources they were taken on, the hash ignores comments, the peak
comes from the measured file, launch counts and the JSON config."""
import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_source_hash_ignores_comments_only(bench, tmp_path):
    a = tmp_path / "a.cu"
    a.write_text("int f() {\n  return 1;  // one\n}\n/* block\n comment */\n")
    b = tmp_path / "b.cu"
    b.write_text("// header\nint f() {\n\n  return 1;   \n}\n")
    c = tmp_path / "c.cu"
    c.write_text("int f() {\n  return 2;\n}\n")
    assert bench.source_hash([str(a)]) == bench.source_hash([str(b)])
    assert bench.source_hash([str(a)]) != bench.source_hash([str(c)])


def test_step_kernel_sources_exist(bench):
    for p in bench.step_kernel_sources():
        assert os.path.exists(p), p


def test_committed_traffic(bench):
    """When the committed counters were taken on the current step-kernel
    sources, the bench reports them. A call moves the algorithmic bytes (K,
    the distinct kept V rows, q/out/tau: about 338 MB at this workload) plus
    the kept lists the scan writes and the gather reads back (with L2 flushed
    before each captured launch) and the gather's 4-byte scores fetched at
    sector granularity: no more than 30% above the algorithmic bytes. After a
    kernel change the counters are dropped until taken again."""
    t = bench.ncu_traffic(bench.step_kernel_sources())
    if t is None:
        pytest.skip("counters were taken on other kernel sources")
    d = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    assert t == d["dram_bytes_per_call"]
    assert d["scan_dram_read_bytes"] >= 268.4e6          # K is read in full
    assert 1.0 < t / 337.6e6 < 1.3


def test_traffic_is_dropped_when_sources_change(bench, tmp_path):
    src = tmp_path / "k.cu"
    src.write_text("int k;\n")
    assert bench.ncu_traffic([str(src)]) is None


def test_measured_peak(bench):
    gbs, kind = bench.measured_peaks()
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        assert kind == "measured" and gbs == float(json.load(open(p))["hbm_gbs"])
    else:
        assert kind == "fallback" and gbs == bench.FALLBACK_HBM_GBS


def test_launch_counts(bench):
    assert bench.kernels_per_call(dense=True, refresh=False) == 2
    assert bench.kernels_per_call(dense=False, refresh=False) == 2
    assert bench.kernels_per_call(dense=False, refresh=True) == 4


def test_aggregate_and_config(bench):
    import synth
    w = synth.WORKLOADS["llama1b_stack16_b8_128k"]
    assert bench.aggregate_value(64, 1000.0, 1) == pytest.approx(64.0)
    assert bench.aggregate_value(64, 1000.0, 4) == pytest.approx(256.0)
    cfg = bench.workload_config(w, 2)
    assert cfg["workload"] == w.name and cfg["global_batch"] == 2 * w.B
    assert bench.rank_workload(w, 0) is w
    assert bench.rank_workload(w, 1).seed != w.seed


def test_r_cycle_and_schedule(bench):
    """The headline is the average over a refresh cycle of R steps: one
    refresh step and R - 1 plain steps; step t refreshes when t mod R == 0."""
    assert bench.r_cycle(1.0, 4.0, 1) == pytest.approx(1e3 / 4.0)
    assert bench.r_cycle(1.0, 4.0, 32) == pytest.approx(32 / (4.0 + 31 * 1.0) * 1e3)
    s = bench.step_schedule(70, 32)
    assert [t for t, f in enumerate(s) if f] == [0, 32, 64]


def test_config_keys_match_between_arms(bench):
    """The reference arm and our arm report the same config keys."""
    import synth
    w = synth.WORKLOADS["qwen1p5b_128k"]
    a = bench.workload_config(w, 1, bench.replicas_for(w))
    assert {"workload", "l2", "timed_region", "N", "R", "global_batch"} <= set(a)
    assert bench.stack_cap(synth.WORKLOADS["ragged_refresh_b16"]) % 128 == 0


def test_spawn_only_outside_torchrun(bench, monkeypatch):
    args = bench.parse(["--gpus", "1"])
    assert bench.spawn_ranks(args, []) is None
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.parse(["--gpus", "2"])
    assert bench.spawn_ranks(args, []) is None

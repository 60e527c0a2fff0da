"""Host-side pieces of bench.py that need no GPU: the algorithmic byte count of a step and the
DRAM-traffic record read from a committed ncu summary (only for the same summary storage type
and only while the kernel's sources are unchanged)."""
import hashlib
import json
import pathlib

import bench
from sparse_kv_cache_summaries_b200 import synth


def test_step_bytes_at_128k_512():
    wl = synth.WORKLOADS["llama8b_128k_b512"]
    fp32 = bench.step_bytes(wl, "fp32")
    fp16 = bench.step_bytes(wl, "fp16")
    # 8 kv-heads x 8192 blocks x (2 x 128 x 4 + 4 x (4 + 1)) bytes of summaries
    assert fp32["summaries"] == 8 * 8192 * 1044
    assert fp16["summaries"] == 8 * 8192 * (2 * 128 * 2 + 4 * 5)
    # 32 selected blocks of 16 bf16 K and V rows per kv-head
    assert fp32["selected_kv"] == fp16["selected_kv"] == 8 * 32 * 16 * 128 * 2 * 2
    assert fp32["step"] == 70541312
    assert fp32["score_stream_kernel"] == 68427776


def _fake_root(tmp_path: pathlib.Path, summary_dtype: str | None) -> pathlib.Path:
    src = tmp_path / "k.cu"
    src.write_text("// kernel source\n")
    rec = {"kernel": "score_stream_kernel", "workload": "w", "dram_bytes_per_launch": 123.0,
           "sources": ["k.cu"], "source_sha256": hashlib.sha256(src.read_bytes()).hexdigest()}
    if summary_dtype is not None:
        rec["summary_dtype"] = summary_dtype
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "score_stream_kernel_w.json").write_text(json.dumps(rec))
    return tmp_path


def test_traffic_record_is_keyed_by_summary_dtype(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", _fake_root(tmp_path, "fp32"))
    assert bench.profile_traffic("score_stream_kernel", "w", "fp32") == 123.0
    assert bench.profile_traffic("score_stream_kernel", "w", "fp16") is None
    assert bench.profile_traffic("score_stream_kernel", "other", "fp32") is None


def test_traffic_record_without_dtype_means_fp32(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", _fake_root(tmp_path, None))
    assert bench.profile_traffic("score_stream_kernel", "w", "fp32") == 123.0
    assert bench.profile_traffic("score_stream_kernel", "w", "fp16") is None


def test_traffic_record_goes_stale_with_the_source(tmp_path, monkeypatch):
    root = _fake_root(tmp_path, "fp32")
    monkeypatch.setattr(bench, "ROOT", root)
    (root / "k.cu").write_text("// kernel source, changed\n")
    assert bench.profile_traffic("score_stream_kernel", "w", "fp32") is None


def test_clock_records_that_cannot_stand():
    ok = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": [], "samples": 30}
    assert not bench.clocks_rejected(ok)
    assert not bench.clocks_rejected({**ok, "sm_mhz": 1300, "reasons": ["sw_power_cap"]})
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clocks_rejected({**ok, "reasons": ["sw_power_cap", r]})
    assert bench.clocks_rejected({**ok, "sm_mhz": 1000})            # a leftover clock lock
    assert not bench.clocks_rejected({"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0})


def test_region_counts_fill_the_clock_window():
    # 20 steps of ~30 us: a 0.6 ms region; at least 50 regions and at least 0.5 s of them
    n = bench.region_counts(0.6)
    assert n >= bench.MIN_REGIONS and n * 0.6e-3 >= bench.MIN_WINDOW_S
    # a long region: the minimum count, capped by the window's upper bound
    assert bench.region_counts(1000.0) == bench.MIN_REGIONS
    assert bench.region_counts(1000.0, min_regions=5, max_window_s=2.0) == 5


def test_reference_arm_reports_the_steps_it_timed(capsys):
    class A:
        workload, budget, steps, warmup, gpus = "tiny", None, 3, 1, 1
    bench.run_reference(A, rank=0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 3
    assert line["cpu_baseline"]["cores"] >= 1
    assert line["value"] == line["cpu_baseline"]["value"] == line["e2e"]["value"]

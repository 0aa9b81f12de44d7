"""Host logic of bench.py that decides whether a run counts: the clock record taken during the timed region
(median and maximum SM clock, throttle reasons), from synthetic nvidia-smi rows (no GPU, no nvidia-smi)."""
import bench


def _sampler(rows, marks):
    s = bench.ClockSampler.__new__(bench.ClockSampler)  # no nvidia-smi process
    s.rows, s.proc, s.marks = rows, None, marks
    return s


def _row(t, sm, reasons=("Not Active",) * 4):
    return (t, [str(sm), "1965", "700.0", *reasons])


def test_clock_summary_uses_the_timed_window():
    rows = [_row(0.5, 1000), _row(1.5, 1965), _row(2.0, 1950), _row(2.5, 1965), _row(9.0, 500)]
    out = _sampler(rows, [1.0, 3.0]).summary()
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0 and out["samples"] == 3
    assert out["reasons"] == []


def test_clock_summary_reports_active_reasons_by_name():
    act = ("Not Active", "Active", "Not Active", "Active")  # hw_thermal_slowdown, sw_power_cap
    rows = [_row(1.0, 1300, act), _row(1.1, 1320)]
    out = _sampler(rows, [0.0, 2.0]).summary()
    assert out["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert out["sm_mhz"] == 1310.0


def test_clock_summary_without_samples():
    out = _sampler([], [0.0, 1.0]).summary()
    assert out["samples"] == 0 and out["sm_mhz"] is None
    assert out["reasons"] == ["no nvidia-smi samples"]


def test_clock_summary_takes_rows_within_one_period_of_a_short_window():
    # a timed region shorter than the sampling period: rows within one period of it count, and say so
    p = bench.ClockSampler.PERIOD_MS / 1e3
    rows = [_row(1.0 - p / 2, 1960), _row(1.001 + p / 2, 1965), _row(5.0, 500)]
    out = _sampler(rows, [1.0, 1.001]).summary()
    assert out["samples"] == 2 and out["sm_mhz"] == 1962.5
    assert out["window"].startswith("timed region +-")


def test_clock_summary_ignores_rows_far_from_the_window():
    # rows seconds away from the timed region say nothing about its clocks
    out = _sampler([_row(5.0, 1800), _row(6.0, 1900)], [0.0, 1.0]).summary()
    assert out["samples"] == 0 and out["reasons"] == ["no nvidia-smi samples"]


def test_reference_arm_prints_the_headline_config():
    assert bench.headline_config(1)["parallelism"] == "replicas1"
    assert bench.headline_config(2)["global_batch"] == 8


def test_roofline_traffic_only_for_the_source_it_was_measured_on(monkeypatch):
    h = bench.attention_source_hash()
    monkeypatch.setattr(bench, "ROOF_TRAFFIC", {"bytes": 123, "source_sha256": h})
    assert bench.roof_traffic() == 123
    monkeypatch.setattr(bench, "ROOF_TRAFFIC", {"bytes": 123, "source_sha256": "0" * 64})
    assert bench.roof_traffic() is None
    monkeypatch.setattr(bench, "ROOF_TRAFFIC", {"bytes": None, "source_sha256": h})
    assert bench.roof_traffic() is None


def test_attention_source_hash_ignores_comment_lines(tmp_path, monkeypatch):
    # the hash covers code lines only: a comment-only edit keeps a traffic figure valid
    src = tmp_path / "k.cu"
    src.write_text("int a;\n// note\nint b;\n")
    monkeypatch.setattr(bench, "_ATTN_SOURCES", (str(src),))  # absolute: os.path.join keeps it as it is
    h0 = bench.attention_source_hash()
    src.write_text("int a;\n  // another note\nint b;\n")
    assert bench.attention_source_hash() == h0
    src.write_text("int a;\nint c;\n")
    assert bench.attention_source_hash() != h0

"""Host-side logic of bench.py that needs no GPU: the summary of the clock record
taken during the timed region, the measured-peak lookup with its fallback, and the
DRAM-traffic record that is only reported while the GEMM sources are unchanged."""
import json
import os
import tempfile

import bench


def _sampler_with(lines):
    s = bench.ClockSampler(0)
    f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
    f.write("\n".join(lines) + "\n")
    f.flush()
    s.file = f
    return s


def test_clock_summary_median_under_load_and_reasons():
    # index, sm, sm max, power, active mask, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    rows = ["0, 1965, 1965, 900.1, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1850, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 345, 1965, 120.0, 0x1, Not Active, Not Active, Not Active, Not Active"]
    out = _sampler_with(rows).summary()
    assert out["sm_mhz"] == 1850.0          # the idle sample (below half of max) is left out
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 4


def test_clock_summary_reports_slowdowns_that_reject_a_run():
    rows = ["0, 1500, 1965, 800.0, 0x48, Active, Not Active, Active, Not Active",
            "0, 1490, 1965, 810.0, 0x28, Not Active, Active, Not Active, Not Active"]
    out = _sampler_with(rows).summary()
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples():
    out = _sampler_with([]).summary()
    assert out["reasons"] == ["unavailable"] and out["sm_mhz"] is None


def test_measured_peaks_file_and_fallback(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.measured_peaks()
    assert src == "fallback" and peaks == {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 7000.0, "bf16_tflops": 1600.0}))
    peaks, src = bench.measured_peaks()
    assert src == "measured" and peaks["bf16_tflops"] == 1600.0


def test_traffic_record_is_tied_to_the_gemm_sources(monkeypatch):
    path = os.path.join(bench.ROOT, "profiles", "gemm_dram_traffic_qwen3_block_m8192.json")
    with open(path) as f:
        rec = json.load(f)
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: rec["gemm_source_sha256"])
    assert bench.recorded_traffic() == rec["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: "0" * 64)
    assert bench.recorded_traffic() is None


def test_gemm_source_digest_covers_the_kernel_files():
    d = bench.kernel_source_digest()
    assert len(d) == 64 and d == bench.kernel_source_digest()

"""Host logic of bench.py that decides what a measurement line reports: the
clock and throttle-reason summary of the nvidia-smi samples taken during the
timed region, and the peak the roofline fraction divides by.  No GPU."""
import json

import bench


def _row(sm, smax=1965, hw="Not Active", hwt="Not Active", swt="Not Active", cap="Not Active"):
    return "0, %s, %s, 990.5, 0x0000000000000000, %s, %s, %s, %s\n" % (sm, smax, hw, hwt, swt, cap)


def test_clock_summary_median_and_no_reasons():
    out = bench.summarize_clock_samples([_row(1965), _row(1950), _row(1800)])
    assert out == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3}


def test_clock_summary_reports_every_active_reason():
    rows = [_row(1965, cap="Active"), _row(1400, hw="Active"), _row(1965, swt="Active"),
            _row(1965, hwt="Active")]
    out = bench.summarize_clock_samples(rows)
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap",
                              "sw_thermal_slowdown"]


def test_clock_summary_skips_malformed_rows():
    rows = ["", "garbage\n", "0, [N/A], 1965, 1, 0x0, Not Active, Not Active, Not Active, Not Active\n",
            _row(1327)]
    out = bench.summarize_clock_samples(rows)
    assert out["samples"] == 1 and out["sm_mhz"] == 1327.0 and out["reasons"] == []
    assert bench.summarize_clock_samples([])["sm_mhz"] is None


def test_measured_peaks_prefers_the_measured_file(tmp_path):
    f = tmp_path / "MEASURED_PEAKS.json"
    f.write_text(json.dumps({"hbm_gbs": 6526.8, "bf16_tflops": 1643.7}))
    assert bench.measured_peaks(str(f)) == (6526.8, "measured")
    assert bench.measured_peaks(str(tmp_path / "absent.json")) == (6650.0, "fallback")
    bad = tmp_path / "bad.json"
    bad.write_text("{")
    assert bench.measured_peaks(str(bad)) == (6650.0, "fallback")

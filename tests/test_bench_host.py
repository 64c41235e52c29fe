"""Host logic of bench.py on CPU: the roofline peak chosen from the sampled clocks, the
clock summary parsed from nvidia-smi's CSV, and the whole-job throughput."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

PEAKS = {"bf16_tflops": 1653.3, "bf16_tflops_sustained": 1396.4, "source": "test"}


@pytest.mark.parametrize("clocks,ms_total,burst", [
    ({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}, 80.0, True),       # at the maximum clock
    ({"sm_mhz": 1867.0, "sm_max_mhz": 1965.0}, 80.0, True),       # 95.0 % of it: still burst
    ({"sm_mhz": 1866.0, "sm_max_mhz": 1965.0}, 80.0, False),      # just below
    ({"sm_mhz": 1462.0, "sm_max_mhz": 1965.0}, 900.0, False),     # power-capped long region
    ({"sm_mhz": None, "sm_max_mhz": None}, 999.0, True),          # no record, under a second
    ({"sm_mhz": None, "sm_max_mhz": None}, 1000.0, False),        # no record, a second or more
    ({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}, 5000.0, True),     # the clock decides, not the length
])
def test_peak_follows_the_sampled_clock(clocks, ms_total, burst):
    peak, use_burst, why = bench.choose_bf16_peak(PEAKS, clocks, ms_total)
    assert use_burst is burst
    assert peak == (PEAKS["bf16_tflops"] if burst else PEAKS["bf16_tflops_sustained"])
    assert "median SM clock" in why


def _summary(tmp_path, lines):
    p = tmp_path / "clocks.csv"
    p.write_text("".join(line + "\n" for line in lines))
    c = bench.ClockSampler("0")
    c.path = str(p)
    out = c.summary()
    assert not p.exists()   # the sample file is removed after reading
    return out


def test_clock_summary_median_under_load_and_reasons(tmp_path):
    idle = "0, 120, 1965, 95.1, 0x0, Not Active, Not Active, Not Active, Not Active"
    busy = "0, {mhz}, 1965, 610.0, 0x4, Not Active, Not Active, Not Active, {cap}"
    lines = [idle, busy.format(mhz=1965, cap="Not Active"), busy.format(mhz=1950, cap="Active"),
             busy.format(mhz=1965, cap="Not Active"), "0, [N/A], [N/A], [N/A], [N/A], x, x, x, x", idle]
    s = _summary(tmp_path, lines)
    # idle samples (below half the highest) are left out of the median
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 6 and s["power_w_max"] == 610.0


def test_clock_summary_names_each_slowdown(tmp_path):
    row = "0, 1500, 1965, 700.0, 0x8, {a}, {b}, {c}, Not Active"
    s = _summary(tmp_path, [row.format(a="Active", b="Not Active", c="Not Active"),
                            row.format(a="Not Active", b="Active", c="Active")])
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert s["sm_mhz"] == 1500.0


def test_clock_summary_without_samples(tmp_path):
    s = _summary(tmp_path, [])
    assert s == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}


def test_whole_job_tokens_per_second():
    assert bench.job_tokens_per_s(4.0, 1) == pytest.approx(bench.TOKENS / 4e-3)
    assert bench.job_tokens_per_s(4.0, 8) == pytest.approx(8 * bench.TOKENS / 4e-3)

"""Host logic of bench.py that runs without a GPU: the nvidia-smi clock
summary keeps only the samples taken during the timed region."""
import datetime
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _row(t, mhz, power_cap="Not Active", thermal="Not Active"):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return (f"{ts}, 0, {mhz}, 1965, 900.0, 0x0000000000000004, Not Active, {thermal}, "
            f"Not Active, {power_cap}")


def test_clock_summary_keeps_the_timed_region():
    t0 = 1_800_000_000.0
    text = "\n".join([
        _row(t0 - 0.08, 1965),                       # before: idle
        _row(t0 + 0.02, 1700, power_cap="Active"),
        _row(t0 + 0.07, 1720, power_cap="Active"),
        _row(t0 + 0.12, 1690),
        _row(t0 + 0.30, 1965, thermal="Active"),      # after: not counted
    ])
    s = bench.parse_clock_rows(text, t0, t0 + 0.15)
    assert s["samples"] == 3 and s["in_timed_region"]
    assert s["sm_mhz"] == 1700 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_falls_back_to_all_samples():
    t0 = 1_800_000_000.0
    text = "\n".join([_row(t0 - 1.0, 1900), _row(t0 + 1.0, 1800, thermal="Active")])
    s = bench.parse_clock_rows(text, t0, t0 + 0.05)       # no sample inside the window
    assert s["samples"] == 2 and not s["in_timed_region"]
    assert s["sm_mhz"] == 1850 and s["reasons"] == ["hw_thermal_slowdown"]
    assert bench.parse_clock_rows("", t0, t0 + 1) is None
    assert bench.parse_clock_rows("garbage line\n", None, None) is None

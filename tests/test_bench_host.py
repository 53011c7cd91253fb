"""Host logic of bench.py that needs no GPU: the clock summary of the timed region."""
from __future__ import annotations

import datetime
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _line(ts, sm, reasons=("Not Active",) * 4):
    # timestamp, index, clocks.sm, clocks.max.sm, power.draw, active mask, 4 reasons
    return ", ".join([ts.strftime("%Y/%m/%d %H:%M:%S.%f")[:-3], "0", str(sm), "1965", "800.0", "0x0", *reasons])


def test_clock_summary_of_nvidia_smi_lines_per_phase():
    c = bench.ClockSampler(0)
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0)
    c.phases = [("warm", t0.timestamp()), ("timed", (t0 + datetime.timedelta(milliseconds=400)).timestamp())]
    c.lines = [_line(t0 - datetime.timedelta(milliseconds=200), 345),  # idle, before the warm pass
               _line(t0 + datetime.timedelta(milliseconds=100), 1950),
               _line(t0 + datetime.timedelta(milliseconds=300), 1900,
                     ("Not Active", "Not Active", "Not Active", "Active")),
               _line(t0 + datetime.timedelta(milliseconds=500), 1960)]
    s = c.summary()
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1950
    assert s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    w = c.summary("warm")
    assert w["samples"] == 2 and w["sm_mhz"] == 1925.0
    t = c.summary("timed")
    assert t["samples"] == 1 and t["sm_mhz"] == 1960 and t["reasons"] == []


def test_clock_summary_of_nvml_samples_and_slowdowns():
    c = bench.ClockSampler(0)
    c.phases = [("timed", 100.0), ("after", 100.02)]
    c.samples = [(99.0, 800.0, 1965.0, frozenset()),
                 (100.005, 1200.0, 1965.0, frozenset({"hw_slowdown", "sw_thermal_slowdown"})),
                 (100.010, 1300.0, 1965.0, frozenset()),
                 (100.5, 1965.0, 1965.0, frozenset())]
    s = c.summary("timed")
    assert s["samples"] == 2
    assert s["sm_mhz"] == 1250.0
    assert s["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert c.summary("after")["samples"] == 1
    c.samples = []
    assert c.summary("timed")["samples"] == 0

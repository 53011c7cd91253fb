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


def test_clock_summary_keeps_samples_from_the_mark_on():
    c = bench.ClockSampler(0)
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0)
    c.mark()
    c.t_mark = t0
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


def test_clock_summary_reports_slowdowns_and_no_samples():
    c = bench.ClockSampler(0)
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0)
    c.t_mark = t0
    c.lines = [_line(t0, 1200, ("Active", "Not Active", "Active", "Not Active"))]
    s = c.summary()
    assert s["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    c.lines = []
    assert c.summary()["samples"] == 0

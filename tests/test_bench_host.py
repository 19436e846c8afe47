"""Host-side pieces of bench.py that need no GPU: the clock summary's timed
window and reason bits, and the roofline peaks' source."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_clock_summary_uses_the_marked_window():
    c = bench.ClockSampler(0)
    c.max_mhz = 1965.0
    # (time, MHz, NVML clock-event reason bits)
    c.samples = [(1.0, 1200.0, 0x40), (2.0, 1965.0, 0x4), (2.2, 1900.0, 0), (3.0, 1800.0, 0)]
    c.marks = {"start": 1.5, "end": 2.5}
    out = c.summary()
    assert out["samples"] == 2 and out["sm_mhz"] == (1965.0 + 1900.0) / 2
    assert out["reasons"] == ["sw_power_cap"]        # the thermal bit fell outside the window
    extra = out["with_following_steps"]
    assert extra["samples"] == 4 and "hw_thermal_slowdown" in extra["reasons"]


def test_clock_summary_without_marks_takes_everything():
    c = bench.ClockSampler(0)
    c.samples = [(1.0, 1965.0, 0), (2.0, 1965.0, 0)]
    out = c.summary()
    assert out["samples"] == 2 and "with_following_steps" not in out


def test_peaks_come_from_the_measured_file():
    pk = bench._peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert pk["src"] == "measured" and pk["hbm"] > 1000 and pk["bf16"] > 100
    else:
        assert pk == dict(hbm=6650.0, bf16=1590.0, src="fallback")

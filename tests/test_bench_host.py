"""Host-side logic of bench.py (no GPU): the clock record it attaches to its line."""
import os
import sys
import threading

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def _sampler_with(samples, source="nvml"):
    c = bench.ClockSampler(0)
    c.source = source
    c._t = threading.Thread(target=lambda: None)
    c._t.start()
    c.samples = list(samples)
    return c


def test_clock_record_median_max_and_reasons():
    rec = _sampler_with([(1965.0, 1965.0, []), (1800.0, 1965.0, ["sw_power_cap"]),
                         (1900.0, 1965.0, [])]).stop()
    assert rec["sm_mhz"] == 1900.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"] and rec["samples"] == 3


def test_clock_record_without_samples():
    rec = _sampler_with([]).stop()
    assert rec["sm_mhz"] is None and rec["samples"] == 0


def test_clock_reason_bits_are_the_nvml_ones():
    # clocks-event reason masks of NVML: power cap, hw slowdown, sw / hw thermal slowdown
    assert dict(bench.ClockSampler.REASONS) == {"sw_power_cap": 0x4, "hw_slowdown": 0x8,
                                                "sw_thermal_slowdown": 0x20,
                                                "hw_thermal_slowdown": 0x40}

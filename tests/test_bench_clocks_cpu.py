"""The bench line's clock record (bench.ClockSampler.summary) from rows
parsed as nvidia-smi prints them (csv, no header, no units): the median SM
clock, the highest max clock, and the throttle reasons reported active."""

import bench


def _rows(*rows):
    return [[x.strip() for x in r.split(",")] for r in rows]


def test_clock_summary_median_max_and_reasons():
    cs = bench.ClockSampler(0)
    cs.samples = _rows("1965, 1965, 820.11, Not Active, Not Active, Not Active, Not Active",
                       "1950, 1965, 990.02, Not Active, Not Active, Not Active, Active",
                       "1965, 1965, 1001.5, Not Active, Not Active, Not Active, Active",
                       "345, 1965, 120.0, Not Active, Not Active, Not Active, Not Active")
    s = cs.summary()
    assert s["sm_mhz"] == 1957.5 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 4


def test_clock_summary_flags_thermal_and_hardware_slowdown():
    cs = bench.ClockSampler(0)
    cs.samples = _rows("1500, 1965, 700, Active, Not Active, Not Active, Not Active",
                       "1400, 1965, 700, Not Active, Active, Active, Not Active")
    assert cs.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples():
    cs = bench.ClockSampler(0)
    cs.samples = _rows("[N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]")
    s = cs.summary()
    assert s["sm_mhz"] is None and s["sm_max_mhz"] is None and s["reasons"] == []

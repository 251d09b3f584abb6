"""The bench's clock record: nvidia-smi rows parsed into the median SM clock under load, the
maximum clock and the throttle reasons, restricted to the timed window (host logic, no GPU)."""
import datetime

import bench

CLK = bench.ClockSampler


def _row(t, sm, power, power_cap="Active", thermal="Not Active"):
    stamp = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    # timestamp, index, clocks.sm, clocks.max.sm, power.draw, active mask, hw, hw thermal, sw thermal, sw power cap
    return f"{stamp}, 0, {sm}, 1965, {power}, 0x0004, Not Active, Not Active, {thermal}, {power_cap}\n"


def test_summary_keeps_only_the_timed_window():
    t0 = 1_800_000_000.0
    lines = [_row(t0 + 0.1 * i, 1965 if i < 10 else 1700, 350) for i in range(20)]
    lines += [_row(t0 + 2.5, 800, 120, thermal="Active")]  # after the window: idle, thermal
    s = CLK.summarise(lines, window=(t0 + 1.0, t0 + 1.9))
    assert s["sm_mhz"] == 1700 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 10


def test_summary_median_under_load_and_all_rows_without_a_window():
    t0 = 1_800_000_000.0
    lines = [_row(t0, 1800, 900), _row(t0 + 0.1, 1700, 950), _row(t0 + 0.2, 600, 100, power_cap="Not Active")]
    s = CLK.summarise(lines)
    assert s["sm_mhz"] == 1750  # the idle sample (100 W) is left out of the median
    assert s["samples"] == 3 and s["reasons"] == ["sw_power_cap"]


def test_summary_falls_back_to_all_rows_when_no_sample_is_inside_the_window():
    t0 = 1_800_000_000.0
    lines = [_row(t0 + 0.1 * i, 1650, 800) for i in range(3)]
    s = CLK.summarise(lines, window=(t0 + 10.0, t0 + 10.3))
    assert s["samples"] == 3 and s["sm_mhz"] == 1650


def test_summary_skips_malformed_rows_and_unreadable_timestamps():
    lines = ["garbage\n", "not a time, 0, 1700, 1965, 500, 0x0, Not Active, Not Active, Not Active, Active\n",
             "x, 0, [N/A], 1965, 500, 0x0, Not Active, Not Active, Not Active, Active\n"]
    s = CLK.summarise(lines, window=(0.0, 1.0))
    assert s["samples"] == 1 and s["sm_mhz"] == 1700  # the unreadable stamp disables the window filter

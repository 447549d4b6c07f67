"""The bench line's clock record, from nvidia-smi rows like those sampled during a timed region
(index, SM clock, max SM clock, power, active-reason mask, then hw_slowdown,
hw_thermal_slowdown, sw_thermal_slowdown and sw_power_cap)."""
import bench

IDLE = "0, 345, 1965, 140.2, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active"
BUSY = "0, 1965, 1965, 780.4, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"
CAPPED = "0, 1830, 1965, 998.7, 0x0000000000000004, Not Active, Not Active, Not Active, Active"
HOT = "0, 1500, 1965, 990.0, 0x0000000000000040, Not Active, Not Active, Active, Not Active"


def test_busy_half_median_and_reasons():
    c = bench.summarize_clocks("\n".join([IDLE, BUSY, CAPPED, BUSY, CAPPED, BUSY]))
    # busier half of (345, 1830, 1830, 1965, 1965, 1965): 1965, 1965, 1965
    assert c == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 6}


def test_thermal_reason_is_reported():
    c = bench.summarize_clocks("\n".join([BUSY, HOT, HOT, CAPPED]) + "\n")
    assert c["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
    assert c["sm_mhz"] == (1830.0 + 1965.0) / 2


def test_unreadable_samples():
    assert bench.summarize_clocks("") is None
    c = bench.summarize_clocks("0, [N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]")
    assert c == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 1}

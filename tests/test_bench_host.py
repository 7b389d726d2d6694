"""CPU: host-side choices of bench.py (the bf16 denominator follows the
sampled clocks)."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

PEAKS = (6546.9, 1676.5, 1374.1, "measured")


def test_burst_peak_at_full_clock():
    r = bench.roofline_tensor(1000.0, {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}, PEAKS)
    assert r["peak"] == 1676.5 and r["frac"] == round(1000 / 1676.5, 4)
    assert r["frac_of_sustained_peak"] == round(1000 / 1374.1, 4)


def test_sustained_peak_only_when_power_capped_and_slow():
    slow = {"sm_mhz": 1330, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    assert bench.roofline_tensor(1000.0, slow, PEAKS)["peak"] == 1374.1
    # Power cap flagged but the clock stayed near its maximum: burst.
    fast = {"sm_mhz": 1900, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    assert bench.roofline_tensor(1000.0, fast, PEAKS)["peak"] == 1676.5
    # Slow clock without the power cap (e.g. a clock lock): still burst.
    locked = {"sm_mhz": 1100, "sm_max_mhz": 1965, "reasons": []}
    assert bench.roofline_tensor(1000.0, locked, PEAKS)["peak"] == 1676.5
    # No clock record at all: burst.
    assert bench.roofline_tensor(1000.0, {"sm_mhz": None, "sm_max_mhz": None, "reasons": []},
                                 PEAKS)["peak"] == 1676.5


def test_nominal_fractions_reported_beside_measured():
    r = bench.roofline_tensor(1125.0, {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}, PEAKS)
    assert r["frac_of_nominal"] == 0.5
    h = bench.roofline_hbm(6000.0, 6546.9, "measured", kernel="k", traffic=None)
    assert h["bound"] == "hbm" and h["frac"] == round(6000 / 6546.9, 4)
    assert h["frac_of_nominal"] == 0.75 and h["kernel"] == "k" and h["traffic"] is None

"""Host-side logic of bench.py: which FP8 peak the GEMM's roofline fraction
uses, the clock-scaled ceiling, and the config both arms print."""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

PEAKS = dict(hbm=6557.4, bf16=1629.0, bf16_sustained=1374.6, source="measured")


def test_full_clock_without_power_cap_uses_the_burst_peak():
    r = bench.gemm_roofline(1900.0, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}, PEAKS)
    assert r["peak"] == 2 * 1629.0
    assert abs(r["frac"] - 1900.0 / 3258.0) < 1e-12
    assert abs(r["frac_other_peak"] - 1900.0 / 2749.2) < 1e-12
    # 148 SMs x 16384 FLOP/clk x 1.965 GHz
    assert abs(r["clock_ceiling"] - 148 * 16384 * 1.965e9 / 1e12) < 1e-9
    assert abs(r["frac_spec"] - 1900.0 / 4500.0) < 1e-12


def test_power_capped_or_slow_clock_uses_the_sustained_peak():
    capped = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    slow = {"sm_mhz": 1700.0, "sm_max_mhz": 1965.0, "reasons": []}
    unknown = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    for c in (capped, slow, unknown):
        r = bench.gemm_roofline(1600.0, c, PEAKS)
        assert r["peak"] == 2 * 1374.6
    assert "clock_ceiling" not in bench.gemm_roofline(1600.0, unknown, PEAKS)
    r = bench.gemm_roofline(1600.0, slow, PEAKS)
    assert abs(r["clock_ceiling"] - 148 * 16384 * 1.7e9 / 1e12) < 1e-9


def test_both_arms_print_the_same_config():
    big = [torch.empty(100 * 2 ** 20, dtype=torch.uint8), torch.empty(40 * 2 ** 20, dtype=torch.uint8)]
    desc = {"workload": "w", "M": 1, "N": 2, "K": 3}
    a = bench.run_config(desc, 1, big)
    b = bench.run_config(dict(desc), 1, [t.clone() for t in big])
    assert a == b and a["l2"].startswith("inputs larger")
    assert bench.run_config(desc, 1, None)["l2"] == "inputs smaller than L2"
    assert desc == {"workload": "w", "M": 1, "N": 2, "K": 3}


def test_targets_name_the_spec_fractions_they_are_measured_against():
    roof = bench.gemm_roofline(2800.0, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}, PEAKS)
    t = bench.targets(roof, 6100.0)
    assert abs(t["gemm"]["frac"] - 2800.0 / 4500.0) < 1e-12 and t["gemm"]["met"]
    assert abs(t["quantizers"]["frac"] - 6100.0 / 8000.0) < 1e-12 and t["quantizers"]["met"]
    t = bench.targets(bench.gemm_roofline(1900.0, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0,
                                                    "reasons": []}, PEAKS), 4500.0)
    assert not t["gemm"]["met"] and not t["quantizers"]["met"]
    assert "4500" in t["gemm"]["measured_against"] and "8000" in t["quantizers"]["measured_against"]

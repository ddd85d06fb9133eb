"""Host-side helpers of bench.py: per-step percentiles and the exponential (MUFU) roof."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_step_stats_percentiles():
    ms = [float(v) for v in range(1, 11)]  # 1 .. 10 ms
    s = bench.step_stats(ms)
    assert s["median_ms"] == 5.5
    assert s["p10_ms"] == pytest.approx(1.9)
    assert s["p90_ms"] == pytest.approx(9.1)
    assert bench.step_stats([2.5]) == {"median_ms": 2.5}
    assert bench.step_stats([]) == {}


def test_exp_roof_arithmetic():
    # 16 ex2 per clock per SM on 148 SMs at 1000 MHz: 2.368e12 per second.  2.368e9 pairs in
    # 2 ms is 1.184e12 per second, half of it.
    r = bench.exp_roof(2.368e9, 2.0, 1000)
    assert r["mufu_peak_per_s"] == pytest.approx(2.368e12, rel=1e-3)
    assert r["exp_per_s"] == pytest.approx(1.184e12, rel=1e-3)
    assert r["frac"] == pytest.approx(0.5, abs=1e-4)
    assert bench.exp_roof(1e9, 1.0, None)["sm_mhz"] == 1965.0

"""bench.py's clock record, without a GPU: the throttle-reason bits are NVML's
own, the median SM clock is taken under load (idle samples dropped), and the
reasons reported are those seen under load."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_reason_bits_are_nvml_definitions():
    N = pytest.importorskip("pynvml")
    names = {"gpu_idle": "GpuIdle", "applications_clocks_setting": "ApplicationsClocksSetting",
             "sw_power_cap": "SwPowerCap", "hw_slowdown": "HwSlowdown", "sync_boost": "SyncBoost",
             "sw_thermal_slowdown": "SwThermalSlowdown", "hw_thermal_slowdown": "HwThermalSlowdown",
             "hw_power_brake_slowdown": "HwPowerBrakeSlowdown", "display_clock_setting": "DisplayClockSetting"}
    for bit, name in bench._REASONS.items():
        assert getattr(N, "nvmlClocksThrottleReason" + names[name]) == bit, name
    assert sum(bench._REASONS) == N.nvmlClocksThrottleReasonAll


def _sampler(samples, max_mhz=1965):
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.ok, s.samples, s.max_mhz = True, samples, max_mhz
    return s


def test_median_and_reasons_under_load_only():
    idle = [(285, 0x1, 0)] * 5
    busy = [(1965, 0x0, 90)] * 6 + [(1950, 0x4, 99)] * 3
    r = _sampler(idle + busy + idle).summary()
    assert r["samples"] == len(busy)
    assert r["sm_mhz"] == 1965 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"]  # gpu_idle is never reported


def test_slowdowns_are_reported_by_name():
    busy = [(1965, 0x0, 90), (1500, 0x8 | 0x40, 90), (1600, 0x20, 90)]
    r = _sampler(busy).summary()
    assert set(r["reasons"]) == {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
    assert r["sm_mhz"] == 1600


def test_all_idle_falls_back_to_every_sample():
    r = _sampler([(285, 0x1, 0), (300, 0x1, 0), (345, 0x1, 0)]).summary()
    assert r["samples"] == 3 and r["sm_mhz"] == 300 and r["reasons"] == []


def test_without_nvml_the_record_says_so():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.ok, s.err = False, "no driver"
    r = s.summary()
    assert r["samples"] == 0 and r["sm_mhz"] is None and "no driver" in r["note"]

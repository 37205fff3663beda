"""The bench's clock record (bench.ClockSampler) on the CPU: only samples taken inside the
timed window count, throttle reasons come from NVML's bit masks, and a window shorter
than one poll still gets the nearest sample."""
import threading

import pytest

import bench


def _sampler(samples, window, max_mhz=1965.0):
    s = bench.ClockSampler(0)
    s.nvml = object()                  # the NVML path, with samples already taken
    s.thread = threading.Thread(target=lambda: None)
    s.thread.start()
    s.samples = list(samples)
    s.window = list(window)
    s.max_mhz = max_mhz
    return s


def test_reason_bits_are_nvmls():
    pynvml = pytest.importorskip("pynvml")
    bits = dict(bench.ClockSampler.REASONS)
    assert bits["sw_power_cap"] == pynvml.nvmlClocksEventReasonSwPowerCap
    assert bits["hw_slowdown"] == pynvml.nvmlClocksEventReasonHwSlowdown
    assert bits["sw_thermal_slowdown"] == pynvml.nvmlClocksEventReasonSwThermalSlowdown
    assert bits["hw_thermal_slowdown"] == pynvml.nvmlClocksEventReasonHwThermalSlowdown


def test_only_the_timed_window_counts():
    idle, cap = 0x1, 0x4  # GPU idle; software power cap
    samples = ([(0.90 + 0.002 * i, 1965.0, idle, 250.0) for i in range(20)] +      # before
               [(1.00 + 0.002 * i, 1600.0 + i, cap, 990.0) for i in range(26)] +   # window
               [(1.10 + 0.002 * i, 1965.0, idle, 400.0) for i in range(20)])       # after
    r = _sampler(samples, (1.0, 1.0505)).stop()
    assert r["samples"] == 26
    assert r["sm_mhz"] == pytest.approx(1612.5)
    assert r["sm_min_mhz"] == 1600.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]        # the idle bit is not a throttle reason
    assert r["power_w"] == 990.0


def test_window_shorter_than_a_poll_takes_the_nearest_sample():
    samples = [(1.000, 1965.0, 0, 300.0), (1.004, 1950.0, 0x8, 310.0)]
    r = _sampler(samples, (1.0031, 1.0032)).stop()
    assert r["samples"] == 1 and r["sm_mhz"] == 1950.0 and r["reasons"] == ["hw_slowdown"]


def test_no_samples_no_record():
    assert _sampler([], (1.0, 2.0)).stop() is None

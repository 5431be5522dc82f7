"""Host logic of bench.py that needs no GPU: the clock record and the launch
timer's choice of how many launches to time (with a stand-in for the CUDA
calls)."""
import time
import types

import torch

import bench


def _row(sm, smax=1965, hw="Not Active", hwt="Not Active", swt="Not Active", cap="Not Active"):
    return f"{sm}, {smax}, 512.3, 0x0000000000000000, {hw}, {hwt}, {swt}, {cap}"


def test_clock_summary_median_and_reasons():
    lines = [_row(1965), _row(1950, cap="Active"), _row(1800), "", "garbage", _row("[N/A]")]
    s = bench.ClockSampler.summary(lines)
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1950
    assert s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_reports_every_throttle_reason():
    s = bench.ClockSampler.summary([_row(1500, hw="Active", hwt="Active", swt="Active")])
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_rows_is_none():
    assert bench.ClockSampler.summary([]) is None
    assert bench.ClockSampler.summary(["a, b"]) is None


class _Event:
    made = 0

    def __init__(self, enable_timing=False):
        _Event.made += 1
        self.t = None

    def record(self, stream):
        self.t = time.perf_counter()

    def elapsed_time(self, other):
        return (other.t - self.t) * 1e3


def _timer():
    clocks = bench.ClockSampler("GPU-test")
    timer = bench.LaunchTimer("cpu", None, clocks)
    timer.torch = types.SimpleNamespace(cuda=types.SimpleNamespace(synchronize=lambda: None, Event=_Event))
    timer.flush_buf = torch.empty(16, dtype=torch.uint8)
    return timer, clocks


def test_launch_timer_fills_the_minimum_timed_region():
    """A 2 ms launch: 0.25 s needs about 125 timed launches, more than the
    20 asked for; the sampler is active only while they run."""
    timer, clocks = _timer()
    calls = []

    def fn():
        calls.append(clocks.active)
        time.sleep(0.002)

    _Event.made = 0
    ms = timer.time(fn, 20, 3)
    timed = _Event.made // 2
    assert 20 < timed <= bench.TIMED_MAX_LAUNCHES
    assert timed * 2e-3 >= 0.5 * bench.TIMED_MIN_S
    assert len(calls) == 3 + bench.TIMED_PROBE + timed
    assert not any(calls[:3 + bench.TIMED_PROBE]) and all(calls[3 + bench.TIMED_PROBE:])
    assert clocks.active is False
    assert 1.5 <= ms <= 50


def test_launch_timer_caps_fast_launches_and_keeps_long_step_counts():
    timer, _ = _timer()
    _Event.made = 0
    timer.time(lambda: None, 20, 3)
    assert _Event.made // 2 == bench.TIMED_MAX_LAUNCHES
    _Event.made = 0
    timer.time(lambda: time.sleep(0.02), 30, 3)
    assert _Event.made // 2 == 30

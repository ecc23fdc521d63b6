"""bench.ClockSampler on the CPU against a fake NVML: samples keep coming while
the launching thread is busy in Python, throttle reasons are collected, and the
interpreter's switch interval is restored afterwards."""
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class FakeNvml:
    NVML_CLOCK_SM = 0

    def __init__(self):
        self.calls = 0

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.calls += 1
        return 1965 if self.calls % 2 else 1900

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return 0x4  # sw_power_cap

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965


def test_sampler_samples_during_a_busy_python_loop(monkeypatch):
    fake = FakeNvml()

    def handle(self):
        self._nvml = fake
        return object()

    monkeypatch.setattr(bench.ClockSampler, "_handle", handle)
    before = sys.getswitchinterval()
    with bench.ClockSampler(0, period_s=0.001) as cs:
        t0 = time.perf_counter()
        x = 0
        while time.perf_counter() - t0 < 0.03:  # 30 ms of pure-Python work
            x += 1
    assert sys.getswitchinterval() == before
    out = cs.summary()
    assert out["samples"] >= 5, out
    assert out["sm_max_mhz"] == 1965 and out["reasons"] == ["sw_power_cap"]
    assert 1900 <= out["sm_mhz"] <= 1965

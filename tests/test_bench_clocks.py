"""The clock record of bench.py on CPU: the nvidia-smi sampler against a fake
sampler process that prints the same CSV lines.

The sampler must come up before the timed region starts. It must count only
the samples from its mark on, report the median SM clock and every active
throttle reason among those samples, and say how many untimed soak steps
were run.
"""
import os
import subprocess
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

_POPEN = subprocess.Popen  # the real one (the tests replace the module attribute)

# one CSV line per sample, in the field order of ClockSampler.FIELDS
IDLE = "345, 1965, 120.5, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active"
LOAD = "1965, 1965, 980.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active"


def _fake_popen(lines_before, lines_after, delay_s):
    """A Popen stand-in running a child process that waits `delay_s`, then
    prints `lines_before`, then keeps printing `lines_after` every 20 ms."""
    script = (
        "import sys, time\n"
        f"time.sleep({delay_s})\n"
        f"for ln in {lines_before!r}: print(ln, flush=True)\n"
        "while True:\n"
        f"    for ln in {lines_after!r}: print(ln, flush=True)\n"
        "    time.sleep(0.02)\n")

    def popen(args, stdout=None, stderr=None):
        assert args[0] == "nvidia-smi" and "-lms" in args
        return _POPEN([sys.executable, "-c", script], stdout=stdout, stderr=stderr)

    return popen


def test_start_waits_for_the_first_sample_and_mark_drops_earlier_ones(monkeypatch):
    monkeypatch.setattr(bench.subprocess, "Popen", _fake_popen([IDLE] * 3, [LOAD], 0.5))
    t0 = time.perf_counter()
    s = bench.ClockSampler("GPU-fake").start()
    assert time.perf_counter() - t0 >= 0.4  # returned only once lines were written
    time.sleep(0.05)
    s.mark()  # the idle lines (and any load line so far) are before the mark
    t1 = time.perf_counter()
    while s.count() < 5 and time.perf_counter() - t1 < 5:
        time.sleep(0.02)
    s.soak_steps = 16
    rec = s.stop()
    assert rec["samples"] >= 5
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["soak_steps"] == 16


def test_reasons_and_median_over_mixed_samples(monkeypatch):
    slow = "1500, 1965, 700.0, 0x0000000000000008, Active, Not Active, Not Active, Not Active"
    monkeypatch.setattr(bench.subprocess, "Popen", _fake_popen([], [LOAD, slow, LOAD], 0.0))
    s = bench.ClockSampler("GPU-fake").start()
    s.mark()
    t1 = time.perf_counter()
    while s.count() < 9 and time.perf_counter() - t1 < 5:
        time.sleep(0.02)
    rec = s.stop()
    assert rec["samples"] >= 9
    assert rec["sm_mhz"] == 1965.0  # two of every three samples at full clock
    assert rec["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_no_sampler_binary_gives_an_unsampled_record(monkeypatch):
    def missing(*a, **k):
        raise FileNotFoundError("nvidia-smi")

    monkeypatch.setattr(bench.subprocess, "Popen", missing)
    s = bench.ClockSampler("GPU-fake").start()
    assert s.count() == 0
    rec = s.stop()
    assert rec["sm_mhz"] is None and rec["reasons"] == ["unsampled"]


if __name__ == "__main__":
    sys.exit(pytest.main([__file__, "-q"]))

"""Host-side parts of bench.py that need no GPU: the clock sampler's
in-process polling and summary (with a fake NVML), and the bounded reference
arm's per-step budget."""
import importlib.util
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    try:
        sys.argv = ["bench.py"]
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


class FakeNvml:
    NVML_CLOCK_SM = 1

    def __init__(self, mhz=1700, reasons=0x4, fail=False):
        self.mhz, self.reasons, self.fail = mhz, reasons, fail

    def nvmlInit(self):
        if self.fail:
            raise RuntimeError("NVML unavailable")

    def nvmlDeviceGetHandleByIndex(self, i):
        return i

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.mhz

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons


def test_clock_polling_until_the_timing_event_completes():
    b = _bench()
    clk = b.ClockSampler(0)
    calls = []
    clk.poll_until(lambda: len(calls.append(1) or calls) > 4, nvml=FakeNvml())
    s = clk.summary()
    assert s["samples"] == 4 and s["sm_mhz"] == 1700 and s["sm_min_mhz"] == 1700
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_polling_never_raises():
    b = _bench()
    clk = b.ClockSampler(0)
    clk.poll_until(lambda: False, nvml=FakeNvml(fail=True))
    assert clk.summary() is None


def test_reference_budget_is_bounded():
    b = _bench()
    src = open(os.path.join(ROOT, "bench.py")).read()
    assert "90.0 / max(1, args.steps + args.warmup)" in src
    assert hasattr(b, "OracleSampler")

"""bench.py's clock sampler on the host, against a fake NVML: it starts NVML
and takes its first sample before the timed region begins, drops that
sample, samples every half millisecond during the region (20 or more
samples in a few tens of milliseconds, with room for a loaded host), and
reports the throttle reasons it saw."""
import importlib.util
import os
import sys
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fake_nvml(clocks):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    state = {"i": 0}
    nv.nvmlInit = lambda: time.sleep(0.05)          # NVML start-up takes a while
    nv.nvmlDeviceGetHandleByIndex = lambda i: ("gpu", i)
    nv.nvmlDeviceGetMaxClockInfo = lambda h, which: 1965

    def clock(h, which):
        v = clocks[min(state["i"], len(clocks) - 1)]
        state["i"] += 1
        return v

    nv.nvmlDeviceGetClockInfo = clock
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4 if state["i"] > 3 else 0   # sw_power_cap
    return nv


def test_clock_sampler_covers_the_region(monkeypatch):
    clocks = [999] + [1650] * 100000                # the first sample is taken before the region
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(clocks))
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    with bench.ClockSampler(0) as c:
        time.sleep(0.04)                            # a region a little longer than the bench's main step
    s = c.summary()
    assert s["samples"] >= 20, s
    assert s["sm_mhz"] == 1650 and s["sm_mhz_min"] == 1650, s     # the pre-region sample is dropped
    assert s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"], s

"""Host-side pieces of bench.py, without a GPU: the clock sampler against a
fake NVML (it starts NVML and takes a first sample before the timed region
begins, drops that sample, samples every half millisecond during the region
-- 20 or more samples in a few tens of milliseconds, with room for a loaded
host -- and reports the throttle reasons it saw), and the hash check that
keeps a committed DRAM-traffic record to the kernel sources it was taken on."""
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


def test_traffic_record_is_used_only_for_the_sources_it_was_taken_on(tmp_path):
    """bench.py reports a committed DRAM-traffic record only while the hash of
    the kernel sources it names matches; after an edit it reports null."""
    import hashlib
    import json
    spec = importlib.util.spec_from_file_location("bench_under_test2", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    rec = {"sources": ["k.cu"], "sources_sha256_16": hashlib.sha256(b"kernel v1\n").hexdigest()[:16],
           "mean_per_launch_bytes": 1234.0}
    (tmp_path / "profiles" / "rec.json").write_text(json.dumps(rec))
    bench.ROOT = str(tmp_path)
    assert bench._traffic("rec.json", "mean_per_launch_bytes") == 1234.0
    src.write_text("kernel v2\n")
    assert bench._traffic("rec.json", "mean_per_launch_bytes") is None
    assert bench._traffic("missing.json", "mean_per_launch_bytes") is None

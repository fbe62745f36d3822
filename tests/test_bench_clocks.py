"""The benchmark's clock sampler on the CPU, against a fake NVML module: its
start-up queries happen on entry, a gated sampler keeps samples only between
on() and off() (it is entered before the warm-up, so its own start-up never
falls into the timed steps), throttle reasons are decoded from the mask, and
a missing NVML reports no clocks rather than guessing. Also the traffic
table's rule: a captured figure only while its sources are unchanged."""

import sys
import threading
import time
import types

import pytest


def _fake_nvml(mhz=1965, watts=250.0, mask=0):
    calls = {"clock": 0}
    lock = threading.Lock()
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByIndex = lambda i: ("handle", i)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        with lock:
            calls["clock"] += 1
        return mhz

    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetPowerUsage = lambda h: int(watts * 1000)
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: mask
    return m, calls


def _wait_for(pred, seconds=2.0):
    t0 = time.time()
    while not pred() and time.time() - t0 < seconds:
        time.sleep(0.002)
    return pred()


def test_gated_sampler_keeps_only_the_timed_region(monkeypatch):
    import bench

    nv, calls = _fake_nvml()
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    with bench.ClockSampler(0, period_s=0.001, gated=True) as c:
        # the first query ran on entry; the thread keeps querying, keeps nothing
        assert calls["clock"] >= 1
        assert _wait_for(lambda: calls["clock"] >= 5)
        assert c.samples == []
        c.on()
        assert _wait_for(lambda: len(c.samples) >= 3)
        c.off()
        time.sleep(0.01)
        kept = len(c.samples)
        time.sleep(0.02)
        assert len(c.samples) == kept  # nothing after off()
    s = c.summary()
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965
    assert s["samples"] == kept and s["reasons"] == []
    assert s["power_w_median"] == pytest.approx(250.0)


def test_ungated_sampler_records_from_the_start_and_decodes_reasons(monkeypatch):
    import bench

    nv, _ = _fake_nvml(mask=0x4 | 0x1)  # power cap, and idle (dropped from the summary)
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    with bench.ClockSampler(0, period_s=0.001) as c:
        assert _wait_for(lambda: len(c.samples) >= 2)
    s = c.summary()
    assert s["reasons"] == ["sw_power_cap"]
    assert s["samples"] >= 2


def test_missing_nvml_reports_no_clocks(monkeypatch):
    import bench

    broken = types.ModuleType("pynvml")

    def fail():
        raise RuntimeError("no NVML here")

    broken.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", broken)
    with bench.ClockSampler(0, gated=True) as c:
        c.on()
        c.off()
    s = c.summary()
    assert s["sm_mhz"] is None and s["samples"] == 0
    assert "no NVML here" in s["error"]


def test_traffic_figure_only_while_the_sources_match(monkeypatch):
    """A captured DRAM-traffic figure is reported only while every source it
    was captured on still hashes to the recorded digest."""
    import hashlib
    import os

    import bench

    path = os.path.join(bench.ROOT, "bwd_causal_sdpa_b200", "csrc", "common.cuh")
    with open(path, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()[:16]
    table = {("k", "w"): (1.5e6, {"common.cuh": digest}),
             ("k", "stale"): (2.5e6, {"common.cuh": "0" * 16})}
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", table)
    assert bench.measured_traffic("k", "w") == 1.5e6
    assert bench.measured_traffic("k", "stale") is None
    assert bench.measured_traffic("k", "unknown") is None

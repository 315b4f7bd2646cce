"""bench.py's clock sampler against a fake NVML (CPU only): samples are taken
in the background, only those inside the marked timed window count, the
median SM clock and the union of the active clock-event reasons are
reported, and no GPU setting is ever written (the fake has no setters)."""
import sys
import time
import types

import bench


def _fake_nvml(clock_seq, reason_seq):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.nvmlClocksEventReasonHwSlowdown = 0x8
    nv.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nv.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nv.nvmlClocksEventReasonSwPowerCap = 0x4
    state = {"i": 0}

    def nxt(seq):
        v = seq[min(state["i"], len(seq) - 1)]
        return v

    def clock(handle, kind):
        v = nxt(clock_seq)
        state["i"] += 1
        return v

    nv.nvmlInit = lambda: None
    nv.nvmlDeviceGetHandleByUUID = lambda uuid: "h"
    nv.nvmlDeviceGetHandleByIndex = lambda i: "h"
    nv.nvmlDeviceGetMaxClockInfo = lambda handle, kind: 1965
    nv.nvmlDeviceGetClockInfo = clock
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda handle: nxt(reason_seq)
    return nv


def test_clock_sampler_reports_the_window_median_and_reasons(monkeypatch):
    clocks = [1200] * 5 + [1965] * 10000
    reasons = [0x8] * 5 + [0x4] * 10000          # hw_slowdown only before the window
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(clocks, reasons))
    cs = bench.ClockSampler(0)
    cs.start()
    time.sleep(0.1)                               # the early samples fall before the window
    cs.mark_start()
    time.sleep(0.15)
    cs.mark_stop()
    time.sleep(0.05)
    cs.stop()
    s = cs.summary()
    assert s["source"] == "nvml"
    assert s["samples"] >= 3
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    # everything sampled, window or not, saw the early hw_slowdown
    assert any("hw_slowdown" in x[3] for x in cs.samples)


def test_clock_sampler_without_samples():
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.samples, cs.t0, cs.t1, cs.source = [], 1.0, 2.0, None
    assert cs.summary()["reasons"] == ["no samples"]

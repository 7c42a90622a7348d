"""The bench's clock record (bench.ClockSampler) against a fake NVML: the median
SM clock of the samples inside the timed region and the clock-event reasons by
their NVML bits.  No GPU: the fake module stands in for pynvml."""
import sys
import time
import types

import bench


def fake_nvml(clocks, reasons):
    """A pynvml stand-in whose SM clock and reason bits follow the given lists
    (one entry per query, the last repeated)."""
    state = {"i": 0}
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByPciBusId = lambda bus: (_ for _ in ()).throw(RuntimeError("no bus"))
    m.nvmlDeviceGetHandleByIndex = lambda i: ("gpu", i)
    m.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965

    def clock(h, c):
        i = min(state["i"], len(clocks) - 1)
        state["i"] += 1
        return clocks[i]

    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons[min(state["i"], len(reasons)) - 1]
    return m


def test_clock_sampler_reads_nvml(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml([1965, 1500, 1400, 1300], [0x0, 0x4, 0x4, 0x4]))
    c = bench.ClockSampler(0)
    with c:
        t0 = c.mark()
        time.sleep(0.1)
        t1 = c.mark()
    s = c.summary(t0, t1)
    assert s["source"] == "nvml"
    assert s["samples"] >= 5                        # every 2 ms over 0.1 s
    assert s["sm_max_mhz"] == 1965
    assert 1300 <= s["sm_mhz"] <= 1500              # most samples sit at the last value
    assert s["reasons"] == ["sw_power_cap"]         # bit 0x4


def test_clock_sampler_maps_every_reported_reason(monkeypatch):
    bits = 0x8 | 0x20 | 0x40 | 0x1                  # hw slowdown, sw/hw thermal, idle (ignored)
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml([1000], [bits]))
    c = bench.ClockSampler(0)
    with c:
        t0 = c.mark()
        time.sleep(0.03)
        t1 = c.mark()
    s = c.summary(t0, t1)
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert s["sm_mhz"] == 1000


def test_clock_sampler_without_nvml_or_smi(monkeypatch):
    bad = types.ModuleType("pynvml")

    def fail():
        raise RuntimeError("no driver")

    bad.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", bad)
    monkeypatch.setattr(bench.subprocess, "Popen",
                        lambda *a, **k: (_ for _ in ()).throw(OSError("no nvidia-smi")))
    c = bench.ClockSampler(0)
    with c:
        t0 = c.mark()
        t1 = c.mark()
    s = c.summary(t0, t1)
    assert s["samples"] == 0 and s["sm_mhz"] is None

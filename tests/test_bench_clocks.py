"""bench.py's clock sampler against a fake NVML (no GPU needed): the median SM
clock, the maximum and the clock-event reasons seen while it runs."""
import sys
import time
import types


def _fake_nvml(clocks, reasons):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlClocksEventReasonSwPowerCap = 0x4
    m.nvmlClocksEventReasonHwSlowdown = 0x8
    m.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    m.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    state = {"i": 0}
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByIndex = lambda i: ("dev", i)
    m.nvmlDeviceGetHandleByUUID = lambda u: ("dev", u)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        state["i"] += 1
        return clocks[(state["i"] - 1) % len(clocks)]
    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons
    return m


def test_nvml_sampler_reports_median_and_reasons(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1800, 1900, 1700], 0x4 | 0x1))
    import bench
    c = bench.Clocks("0")
    c.start()
    time.sleep(0.1)
    r = c.stop()
    assert r["samples"] >= 3
    assert r["sm_mhz"] in (1700, 1800, 1900)
    assert r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"]       # bit 0x1 (idle) is not a reason we report


def test_throttle_reasons_are_named():
    import bench
    assert set(bench.Clocks.NAMES) == {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                       "sw_power_cap"}

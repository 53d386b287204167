"""The bench's clock sampling on CPU: the nvidia-smi row parser on captured
rows, the under-load summary, and the NVML sampling thread against a fake
NVML module (read-only queries only)."""
import sys
import time
import types

import bench


def test_parse_smi_rows():
    # captured rows of `--query-gpu=clocks.sm,clocks.max.sm,power.draw,<4 reasons> --format=csv,noheader,nounits`
    x = bench.parse_smi_row("1965, 1965, 264.01, Not Active, Not Active, Not Active, Active")
    assert x == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "power_w": 264.01, "reasons": ["sw_power_cap"]}
    y = bench.parse_smi_row("1365, 1965, 994.26, Active, Not Active, Not Active, Not Active")
    assert y["reasons"] == ["hw_slowdown"] and y["sm_mhz"] == 1365.0
    z = bench.parse_smi_row("1965, 1965, [N/A]")                      # clocks only, power unreadable
    assert z["reasons"] == [] and z["power_w"] is None
    assert bench.parse_smi_row("[Unknown Error]") is None


def test_summary_uses_samples_under_load():
    s = [{"sm_mhz": 345.0, "sm_max_mhz": 1965.0, "power_w": 120.0, "reasons": []},
         {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "power_w": 700.0, "reasons": []},
         {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "power_w": 990.0, "reasons": ["sw_power_cap"]},
         {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "power_w": 800.0, "reasons": []}]
    out = bench.summarise_clocks(s)
    assert out["sm_mhz"] == 1965.0 and out["samples"] == 4 and out["samples_under_load"] == 3
    assert out["reasons"] == ["sw_power_cap"] and out["power_w_max"] == 990.0
    assert bench.summarise_clocks([], "nvml: x")["reasons"] == ["no samples: nvml: x"]


def _fake_nvml(calls):
    N = types.ModuleType("pynvml")
    N.NVML_CLOCK_SM = 1
    N.nvmlClocksEventReasonHwSlowdown = 0x8
    N.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    N.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    N.nvmlClocksEventReasonSwPowerCap = 0x4

    class NVMLError(Exception):
        pass
    N.NVMLError = NVMLError
    N.nvmlInit = lambda: calls.append("init")
    N.nvmlShutdown = lambda: calls.append("shutdown")

    def by_bus(b):
        calls.append(("bus", b))
        return "h"
    N.nvmlDeviceGetHandleByPciBusId = by_bus
    N.nvmlDeviceGetClockInfo = lambda h, c: 1965
    N.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    N.nvmlDeviceGetPowerUsage = lambda h: 512000
    N.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4
    N.nvmlDeviceGetUtilizationRates = lambda h: types.SimpleNamespace(gpu=100)
    return N


def test_nvml_thread_samples_and_windows(monkeypatch):
    calls = []
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(calls))
    c = bench.Clocks("00000000:1B:00.0", period=0.01).start()
    t0 = time.perf_counter()
    time.sleep(0.15)
    t1 = time.perf_counter()
    out = c.stop()
    assert ("bus", b"00000000:1B:00.0") in calls and calls[-1] == "shutdown"
    assert out["samples"] >= 3 and out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"] and out["power_w_max"] == 512.0
    w = c.window(t0, t1)
    assert 1 <= w["samples"] <= out["samples"]

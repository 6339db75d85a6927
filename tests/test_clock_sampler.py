"""bench.py's clock sampler against a fake NVML (read-only queries), on CPU."""
import os
import sys
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fake_nvml(clocks, reasons_bits):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlClocksEventReasonSwPowerCap = 0x4
    m.nvmlClocksEventReasonHwSlowdown = 0x8
    m.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    m.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    m.nvmlClocksEventReasonHwPowerBrakeSlowdown = 0x80
    state = {"i": 0, "init": 0}
    m.nvmlInit = lambda: state.__setitem__("init", state["init"] + 1)
    m.nvmlDeviceGetHandleByUUID = lambda u: ("uuid", u)
    m.nvmlDeviceGetHandleByIndex = lambda i: ("index", i)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        state["i"] += 1
        return clocks[state["i"] % len(clocks)]
    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons_bits
    return m, state


def _sample(fake, seconds=0.05):
    sys.path.insert(0, ROOT)
    import bench
    import torch
    saved = sys.modules.get("pynvml")
    sys.modules["pynvml"] = fake
    try:
        c = bench.ClockSampler(torch.device("cuda", 0))
        with c:
            time.sleep(seconds)
        return c.summary()
    finally:
        if saved is None:
            del sys.modules["pynvml"]
        else:
            sys.modules["pynvml"] = saved


def test_samples_and_median_clock():
    fake, state = _fake_nvml([1965, 1965, 1800], 0)
    s = _sample(fake)
    assert state["init"] == 1
    assert s["source"].startswith("nvml")
    assert s["samples"] >= 5
    assert s["sm_mhz"] in (1965.0, 1800.0) and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == []


def test_reasons_are_decoded_from_the_bitmask():
    fake, _ = _fake_nvml([1500], 0x4 | 0x40)
    s = _sample(fake)
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert s["sm_mhz"] == 1500.0


def test_no_nvml_and_no_smi_reports_unavailable(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    import subprocess
    import torch

    broken = types.ModuleType("pynvml")                  # import works, init fails

    def fail():
        raise RuntimeError("no driver")
    broken.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", broken)

    def no_smi(*a, **k):
        raise FileNotFoundError("nvidia-smi")
    monkeypatch.setattr(subprocess, "Popen", no_smi)
    c = bench.ClockSampler(torch.device("cuda", 0))
    with c:
        pass
    s = c.summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None and "unavailable" in s["source"]

"""bench.py's clock sampler against a fake NVML (no GPU): the clocks, power and throttle reasons
it reports, and its fallbacks."""
import importlib.util
import os
import sys
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _fake_nvml(reason_bits, sm=1950, max_sm=1965, milliwatts=700000):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    calls = {"init": 0, "shutdown": 0, "uuid": None}

    def init():
        calls["init"] += 1

    def shutdown():
        calls["shutdown"] += 1

    def by_uuid(u):
        calls["uuid"] = u
        return "handle"

    m.nvmlInit = init
    m.nvmlShutdown = shutdown
    m.nvmlDeviceGetHandleByUUID = by_uuid
    m.nvmlDeviceGetHandleByIndex = lambda i: "handle"
    m.nvmlDeviceGetMaxClockInfo = lambda h, c: max_sm
    m.nvmlDeviceGetClockInfo = lambda h, c: sm
    m.nvmlDeviceGetPowerUsage = lambda h: milliwatts
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reason_bits
    return m, calls


def _sample(monkeypatch, fake, seconds=0.03, gpu="GPU-1234"):
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    bench = _bench()
    with bench.ClockSampler(gpu) as clk:
        time.sleep(seconds)
    return clk.summary()


def test_nvml_samples_a_short_region_densely(monkeypatch):
    fake, calls = _fake_nvml(0x1 | 0x4)  # idle bit (ignored) and sw_power_cap
    s = _sample(monkeypatch, fake)
    assert s["samples"] >= 5  # a 30 ms region: far more than one nvidia-smi sample
    assert s["sm_mhz"] == 1950 and s["sm_max_mhz"] == 1965 and s["power_w_max"] == 700.0
    assert s["reasons"] == ["sw_power_cap"]
    assert s["source"].startswith("nvml")
    assert calls["uuid"] == "GPU-1234" and calls["init"] == 1 and calls["shutdown"] == 1


def test_slowdown_reasons_are_reported(monkeypatch):
    fake, _ = _fake_nvml(0x8 | 0x40 | 0x20)
    s = _sample(monkeypatch, fake)
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_no_nvml_and_no_nvidia_smi_gives_unsampled(monkeypatch):
    fake = types.ModuleType("pynvml")

    def no_driver():
        raise RuntimeError("no NVIDIA driver")

    fake.nvmlInit = no_driver
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    bench = _bench()

    def no_smi(*a, **k):
        raise FileNotFoundError("nvidia-smi")

    monkeypatch.setattr(bench.subprocess, "Popen", no_smi)
    with bench.ClockSampler("0") as clk:
        pass
    assert clk.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}


def test_unsupported_query_falls_back_to_nvidia_smi(monkeypatch):
    fake, calls = _fake_nvml(0)

    def unsupported(h):
        raise RuntimeError("NVML_ERROR_NOT_SUPPORTED")

    fake.nvmlDeviceGetCurrentClocksEventReasons = unsupported
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    bench = _bench()
    started = []

    class FakeSmi:
        def __init__(self, cmd, stdout=None, stderr=None):
            started.append(cmd)
            stdout.write("0, 1900, 1965, 650.0, 0x4, Not Active, Not Active, Not Active, Active\n")
            stdout.flush()

        def send_signal(self, sig):
            pass

        def wait(self, timeout=None):
            return 0

    monkeypatch.setattr(bench.subprocess, "Popen", FakeSmi)
    with bench.ClockSampler("GPU-1234") as clk:
        pass
    s = clk.summary()
    assert calls["shutdown"] == 1 and started and started[0][0] == "nvidia-smi"
    assert s["sm_mhz"] == 1900 and s["reasons"] == ["sw_power_cap"] and s["source"].startswith("nvidia-smi")

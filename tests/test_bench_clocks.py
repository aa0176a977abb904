"""bench.py's clock record, on CPU: the NVML sampler that reads the SM clock,
power and clock-event reasons during the timed region, driven by a fake
NVML module (the real one needs a GPU).  The sampler only reads."""
import sys
import time
import types

import bench


def _fake_nvml(clocks, reasons, fail_init=False):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    state = {"i": 0}

    def init():
        if fail_init:
            raise RuntimeError("no NVML")

    def clock(h, kind):
        assert kind == m.NVML_CLOCK_SM
        v = clocks[min(state["i"], len(clocks) - 1)]
        state["i"] += 1
        return v

    m.nvmlInit = init
    m.nvmlDeviceGetHandleByIndex = lambda i: ("index", i)
    m.nvmlDeviceGetHandleByUUID = lambda u: ("uuid", u)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons
    m.nvmlDeviceGetPowerUsage = lambda h: 512000  # milliwatts
    return m


def _sample(monkeypatch, fake, gpu="0"):
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    s = bench.NvmlSampler(gpu, period_s=0.001)
    with s:
        time.sleep(0.05)
    return s.summary()


def test_nvml_sampler_records_clocks_power_and_reasons(monkeypatch):
    out = _sample(monkeypatch, _fake_nvml([1965, 1950, 1965], 0x4 | 0x40))
    assert out["samples"] >= 3
    assert out["sm_max_mhz"] == 1965 and out["sm_mhz"] in (1950, 1965)
    assert out["power_w_max"] == 512.0
    assert out["reasons"] == ["sw_power_cap", "hw_thermal_slowdown"]


def test_nvml_sampler_no_reasons_and_uuid_devices(monkeypatch):
    out = _sample(monkeypatch, _fake_nvml([1965], 0x0), gpu="GPU-1234")
    assert out["reasons"] == [] and out["samples"] >= 1


def test_nvml_sampler_without_nvml_has_no_samples(monkeypatch):
    assert _sample(monkeypatch, _fake_nvml([1965], 0, fail_init=True)) is None


def test_nvml_sampler_summary_starts_at_the_mark(monkeypatch):
    # idle clocks while the sampler starts and the warm-up runs, load clocks
    # after the mark: only the latter count
    clocks = [300] * 20 + [1965] * 10000
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(clocks, 0))
    s = bench.NvmlSampler("0", period_s=0.001)
    with s:
        while len(s.rows) < 25:
            time.sleep(0.001)
        s.mark()
        time.sleep(0.03)
    out = s.summary()
    assert out["sm_mhz"] == 1965 and out["samples"] >= 1
    assert all(r[0] == 1965 for r in s.rows[s._first:])

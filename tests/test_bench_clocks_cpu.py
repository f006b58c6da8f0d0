"""bench.ClockSampler on the CPU: the clock-event reason bits it decodes are
NVML's published ones, a run's reasons and median SM clock come out of NVML
samples (a fake NVML module here, read-only calls only), and the nvidia-smi
fallback parses its CSV lines the same way."""
import sys
import time
import types

import pytest

import bench

pynvml = pytest.importorskip("pynvml")


def test_reason_bits_are_nvmls():
    want = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
            "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
            "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
            "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
    assert dict(bench.ClockSampler.REASONS) == want


def _fake_nvml(samples, max_mhz):
    """A module with the read-only NVML calls ClockSampler makes; it yields
    the given (SM MHz, reason bits) samples, then repeats the last."""
    it = iter(samples)
    last = [samples[0]]

    def cur():
        try:
            last[0] = next(it)
        except StopIteration:
            pass
        return last[0]

    state = {}
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = pynvml.NVML_CLOCK_SM
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByIndex = lambda i: ("gpu", i)
    m.nvmlDeviceGetMaxClockInfo = lambda h, c: max_mhz

    def clock(h, c):
        state["cur"] = cur()
        return state["cur"][0]

    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: state["cur"][1]
    return m


def test_nvml_samples(monkeypatch):
    cap = pynvml.nvmlClocksEventReasonSwPowerCap
    hw = pynvml.nvmlClocksEventReasonHwSlowdown
    idle = pynvml.nvmlClocksEventReasonGpuIdle
    samples = [(1965.0, 0), (1900.0, cap), (1800.0, cap | idle), (1965.0, 0), (1700.0, hw)]
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(samples, 1965))
    cs = bench.ClockSampler(0)
    cs.start()
    t0 = time.time()
    while len(cs.samples) < len(samples) and time.time() - t0 < 5.0:
        time.sleep(0.005)
    out = cs.stop()
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap"]  # idle is not a reason kept
    assert out["samples"] >= len(samples)
    assert out["source"].startswith("nvml")
    # the five samples' median is 1900; repeats of the last one (1700) pull it to 1800 or 1700
    assert out["sm_mhz"] in (1700.0, 1800.0, 1900.0)


def test_no_reason_in_plain_samples(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([(1965.0, 0)], 1965))
    cs = bench.ClockSampler(0)
    cs.start()
    out = cs.stop()
    assert out["reasons"] == [] and out["sm_mhz"] == 1965.0


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_nvidia_smi_lines():
    cs = bench.ClockSampler(0)
    cs.proc = _DoneProc()
    # index, clocks.sm, clocks.max.sm, power, active bits, hw, hw thermal, sw thermal, sw power cap
    cs.lines = ["0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
                "0, 1830, 1965, 998.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
                "0, 1800, 1965, 999.2, 0x0000000000000024, Not Active, Not Active, Active, Active",
                "garbled",
                "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active"]
    out = cs.stop()
    assert out["samples"] == 3 and out["sm_mhz"] == 1830.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
    assert out["source"].startswith("nvidia-smi")

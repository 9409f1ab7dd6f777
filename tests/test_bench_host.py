"""Host logic of the bench on CPU: the clock sampler against a fake NVML,
and the rule that ties the reported DRAM traffic to the profiled kernel
source."""
import re
import sys
import time
import types

import bench


def _fake_nvml(clocks, reasons, max_mhz=1965, fail_init=False):
    it = iter(clocks)
    last = [clocks[-1]]

    def clock(h, which):
        assert which == 1
        try:
            last[0] = next(it)
        except StopIteration:
            pass
        return last[0]

    def init():
        if fail_init:
            raise RuntimeError("NVML not available")

    return types.SimpleNamespace(NVML_CLOCK_SM=1, nvmlInit=init, nvmlDeviceGetHandleByIndex=lambda i: ("gpu", i),
                                 nvmlDeviceGetMaxClockInfo=lambda h, which: max_mhz,
                                 nvmlDeviceGetClockInfo=clock,
                                 nvmlDeviceGetCurrentClocksEventReasons=lambda h: reasons)


def test_clock_sampler_reports_median_max_and_reasons(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1800, 1830, 1860], 0x4 | 0x8))
    with bench.ClockSampler(0, period=0.001) as cs:
        time.sleep(0.05)
    s = cs.summary()
    assert s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert s["samples"] >= 3 and s["sm_mhz"] == 1860        # the last clock repeats after the first three


def test_clock_sampler_without_nvml_reports_nothing(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1800], 0, fail_init=True))
    with bench.ClockSampler(0, period=0.001) as cs:
        time.sleep(0.01)
    assert cs.summary() is None


def test_profiled_traffic_follows_the_kernel_source(monkeypatch):
    """The committed ncu summary's DRAM bytes are reported only while the
    kernel source hash written in it matches the sources."""
    txt = open(bench.os.path.join(bench.ROOT, "profiles", "adam8_step_kernel_llama_layer_m8.md")).read()
    recorded = re.search(r"kernel source hash: `([0-9a-f]+)`", txt).group(1)
    per_launch = float(re.search(r"dram bytes per launch: ([0-9.eE+]+)", txt).group(1))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: recorded)
    assert bench.profiled_traffic("llama_layer_m8", None) == per_launch
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.profiled_traffic("llama_layer_m8", None) is None
    assert bench.profiled_traffic("no_such_workload", None) is None

"""Host logic of bench.py that needs no GPU: the decoding of the clock-event
reasons the timing rules act on (an NVML stand-in feeds the sampler; no GPU
setting is read or changed), the workload config and the selector byte
counts."""
import threading
import time

import pytest

import bench
from synthetic import workload


class _FakeNVML:
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, reasons):
        self.clocks, self.reasons, self.i = clocks, reasons, 0

    def nvmlDeviceGetClockInfo(self, h, kind):
        assert kind == self.NVML_CLOCK_SM
        c = self.clocks[self.i % len(self.clocks)]
        self.i += 1
        return c

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons


def _sample(clocks, reasons, seconds=0.08):
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples, s.reasons, s.max_mhz = [], set(), 1965
    s._stop = threading.Event()
    s._h = object()
    s._nv = _FakeNVML(clocks, reasons)
    with s:
        time.sleep(seconds)
    return s.summary()


def test_power_cap_is_reported_and_idle_ignored():
    out = _sample([1837, 1852, 1845], 0x4 | 0x1)
    assert out["reasons"] == ["sw_power_cap"]
    assert out["sm_max_mhz"] == 1965 and 1837 <= out["sm_mhz"] <= 1852
    assert out["samples"] >= 3


@pytest.mark.parametrize("bits,names", [
    (0x8, ["hw_slowdown"]),
    (0x40 | 0x20, ["hw_thermal_slowdown", "sw_thermal_slowdown"]),
    (0x80, ["hw_power_brake_slowdown"]),
    (0x0, []),
])
def test_slowdown_reasons_decode(bits, names):
    assert _sample([1965], bits)["reasons"] == names


def test_no_nvml_reports_unavailable():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples, s.reasons, s.max_mhz = [], set(), None
    s._stop, s._h = threading.Event(), None
    with s:
        pass
    assert s.summary()["reasons"] == ["unavailable"]


@pytest.mark.parametrize("name", bench.WORKLOADS)
def test_config_names_the_workload_without_model_keys(name):
    c = bench.config_of(workload(name))
    assert c["workload"] == name
    assert not {"model", "global_batch", "seq_len"} & set(c)
    assert "MB flush" in c["l2"]


def test_selector_bytes():
    w = workload("tra_entropy")
    h, N, d = w["heads"], w["N"], w["d"]
    b, bound = bench.selector_bytes(w, 100)
    assert (b, bound) == (2 * h * N * d * 2 + 400, "hbm")  # q and k once, 4 B per entry
    b, bound = bench.selector_bytes(workload("wan_radial"), 36696)
    assert (b, bound) == (4 * 36696, "launch")

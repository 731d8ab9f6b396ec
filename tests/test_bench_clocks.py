"""bench.py's clock sampler on the CPU, against a fake NVML: samples taken
during the region, median / max / throttle-reason summary, and only read-only
queries issued."""
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class FakeNvml:
    """The subset of pynvml the sampler may call; records every name it is asked for."""

    NVML_CLOCK_SM = 1
    QUERIES = {"nvmlInit", "nvmlDeviceGetHandleByPciBusId", "nvmlDeviceGetHandleByIndex",
               "nvmlDeviceGetClockInfo", "nvmlDeviceGetMaxClockInfo",
               "nvmlDeviceGetCurrentClocksEventReasons", "NVML_CLOCK_SM"}

    def __init__(self, clocks, reasons):
        self.used = set()
        self._clocks = list(clocks)
        self._reasons = list(reasons)
        self._i = 0

    def __getattribute__(self, name):
        if not name.startswith("_") and name not in ("used", "QUERIES"):
            object.__getattribute__(self, "used").add(name)
        return object.__getattribute__(self, name)

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        return ("bus", bus)

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("idx", i)

    def nvmlDeviceGetClockInfo(self, h, kind):
        assert kind == 1
        v = self._clocks[min(self._i, len(self._clocks) - 1)]
        return v

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        v = self._reasons[min(self._i, len(self._reasons) - 1)]
        self._i += 1
        return v


def test_sampler_summary_from_fake_nvml():
    fake = FakeNvml(clocks=[1965, 1900, 1750, 1750, 1750, 1800] + [1750] * 100,
                    reasons=[0x0, 0x4, 0x4, 0x1, 0x0] + [0x4] * 100)
    with bench.ClockSampler(0, period_s=0.002, nvml=fake) as clk:
        time.sleep(0.15)
    s = clk.summary()
    assert s["source"] == "nvml"
    assert s["samples"] >= 10                      # first sample + the polls in the region
    assert s["sm_max_mhz"] == 1965.0
    assert s["sm_mhz"] == 1750.0                   # the median under load
    assert s["reasons"] == ["sw_power_cap"]        # idle (0x1) is not a throttle reason
    assert fake.used <= FakeNvml.QUERIES, fake.used - FakeNvml.QUERIES


def test_sampler_names_every_rejecting_reason():
    fake = FakeNvml(clocks=[1965], reasons=[0x8 | 0x20 | 0x40 | 0x80])
    with bench.ClockSampler(0, period_s=0.002, nvml=fake) as clk:
        time.sleep(0.02)
    assert clk.summary()["reasons"] == ["hw_power_brake_slowdown", "hw_slowdown",
                                        "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_sampler_without_any_source_reports_no_samples(monkeypatch):
    class Broken:
        def nvmlInit(self):
            raise RuntimeError("no NVML")

    monkeypatch.setattr(bench.subprocess, "Popen",
                        lambda *a, **k: (_ for _ in ()).throw(FileNotFoundError("nvidia-smi")))
    with bench.ClockSampler(0, nvml=Broken()) as clk:
        pass
    assert clk.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

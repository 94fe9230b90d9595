"""Host logic of bench.py without a GPU: the algorithmic byte counts behind the
roofline, and the clock sampler against a fake NVML (read-only calls)."""
import sys
import time
import types

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402
import workloads as W  # noqa: E402


def test_decode_bytes_of_the_headline_layer():
    """32 x 8192 tokens x 8 kv heads x 146 B per token-head of records (2336 B per
    16-token record), q in bf16, one int32 table entry per block read, fp32 output."""
    w = W.make("qwen3_8b_layer")
    records = 32 * 8192 * 8 * 2336 // 16
    assert bench.decode_kv_bytes(w) == records == 306_184_192
    assert bench.decode_bytes(w) == records + 32 * 32 * 128 * 2 + 32 * 512 * 4 + 32 * 32 * 128 * 4
    assert bench.decode_bytes(w) == 307_036_160


def test_append_bytes_of_the_prefill_chunk():
    """Per token and kv head: bf16 key and value rows in, one record's share out (74 B
    at d 64), plus the int32 slot."""
    w = W.make("prefill_small_head")
    T = 16 * 2048
    assert bench.append_bytes(w, T) == T * 2 * (2 * 64 * 2 + 1184 // 16) + T * 4


def _fake_nvml(clocks, reasons, fail=False):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 0
    m.nvmlClocksEventReasonHwSlowdown = 0x8
    m.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    m.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    m.nvmlClocksEventReasonSwPowerCap = 0x4
    m.nvmlClocksEventReasonHwPowerBrakeSlowdown = 0x80
    it = {"i": 0}

    def init():
        if fail:
            raise RuntimeError("no driver")

    def clock(h, kind):
        it["i"] += 1
        return clocks[it["i"] % len(clocks)]

    m.nvmlInit = init
    m.nvmlDeviceGetHandleByPciBusId = lambda bus: ("handle", bus)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons
    return m


def _sample(monkeypatch, nvml):
    monkeypatch.setitem(sys.modules, "pynvml", nvml)
    with bench.ClockSampler("00000000:00:00.0") as cs:
        cs.mark_start()
        time.sleep(0.05)
        cs.mark_end()
    return cs.summary()


def test_clock_sampler_reports_median_and_reasons(monkeypatch):
    s = _sample(monkeypatch, _fake_nvml([1965, 1965, 1950], 0x4))
    assert s["sm_max_mhz"] == 1965 and s["sm_mhz"] in (1950, 1965) and s["samples"] >= 1
    assert s["reasons"] == ["sw_power_cap"]
    s = _sample(monkeypatch, _fake_nvml([1200], 0x8 | 0x20))
    assert s["sm_mhz"] == 1200 and s["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    s = _sample(monkeypatch, _fake_nvml([1965], 0))
    assert s["reasons"] == []


def test_clock_sampler_without_nvml_reports_it(monkeypatch):
    s = _sample(monkeypatch, _fake_nvml([1965], 0, fail=True))
    assert s["sm_mhz"] is None and s["reasons"][0].startswith("nvml unavailable")

"""Host-side logic of bench.py that needs no GPU: the clock sampler, run
against a fake NVML module in the child process it starts."""
import time

import pytest

FAKE_NVML = '''
NVML_CLOCK_SM = 1
_n = [0]
def nvmlInit():
    pass
def nvmlDeviceGetHandleByPciBusId(bus):
    assert bus == "00000000:1B:00.0", bus
    return "h"
def nvmlDeviceGetMaxClockInfo(h, kind):
    return 1965
def nvmlDeviceGetClockInfo(h, kind):
    _n[0] += 1
    return 1900 if _n[0] % 2 else 1800
def nvmlDeviceGetCurrentClocksEventReasons(h):
    return 0x4 | 0x1
'''


def test_clock_sampler_reads_clocks_and_reasons(tmp_path, monkeypatch):
    (tmp_path / "pynvml.py").write_text(FAKE_NVML)
    monkeypatch.setenv("PYTHONPATH", str(tmp_path))
    import bench

    c = bench.ClockSampler(0)
    monkeypatch.setattr(c, "_bus_id", lambda: "00000000:1B:00.0")
    c.start()
    assert c.poller is not None
    time.sleep(0.05)
    out = c.stop()
    assert out["source"] == "nvml"
    assert out["sm_max_mhz"] == 1965
    assert out["sm_mhz"] in (1800, 1900)
    assert out["reasons"] == ["sw_power_cap"]
    assert out["samples"] >= 5


def test_clock_sampler_without_nvml_returns_none(tmp_path, monkeypatch):
    (tmp_path / "pynvml.py").write_text("def nvmlInit():\n    raise RuntimeError('no driver')\n")
    monkeypatch.setenv("PYTHONPATH", str(tmp_path))
    monkeypatch.setenv("PATH", str(tmp_path))  # no nvidia-smi either
    import bench

    c = bench.ClockSampler(0)
    monkeypatch.setattr(c, "_bus_id", lambda: "00000000:1B:00.0")
    c.start()
    assert c.poller is None
    assert c.stop() is None

"""bench.py's clock record: only samples inside the timed region count, and
the reason bits map to nvidia-smi's names (CPU, no GPU or NVML needed)."""
import importlib.util
import os
import threading

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_samples_outside_the_window_are_dropped():
    B = _bench()
    c = B.ClockSampler(0)
    c.nvml = object()                  # as if NVML had started
    c.t = threading.Thread(target=lambda: None)
    c.t.start()
    c.max_mhz = 1965.0
    c.samples = [(0.5, 1200.0, 0x1),   # idle, before the region
                 (1.0, 1965.0, 0x0), (1.1, 1950.0, 0x4), (1.2, 1965.0, 0x0),
                 (2.5, 800.0, 0x40)]   # after the region
    r = c.stop(1.0, 2.0)
    assert r["samples"] == 3 and r["sm_mhz"] == 1965.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"] and r["source"] == "nvml"


def test_reason_bits():
    B = _bench()
    c = B.ClockSampler(0)
    c.nvml = object()
    c.t = threading.Thread(target=lambda: None)
    c.t.start()
    c.samples = [(1.0, 1000.0, 0x8 | 0x20 | 0x40)]
    r = c.stop(0.0, 2.0)
    assert r["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_no_sampler_available():
    B = _bench()
    r = B.ClockSampler(0).stop(0.0, 1.0)
    assert r["samples"] == 0 and r["sm_mhz"] is None

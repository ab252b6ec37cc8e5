"""Host logic of bench.py that needs no GPU: the nvidia-smi clock summary."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_clock_summary_keeps_the_device_and_collects_reasons():
    b = _bench()
    cs = b.ClockSampler("GPU-aaaa")
    cs.lines = [
        "GPU-bbbb, 1200, 1965, 500.0, Not Active, Not Active, Not Active, Active\n",
        "GPU-aaaa, 1965, 1965, 900.0, Not Active, Not Active, Not Active, Active\n",
        "GPU-aaaa, 1950, 1965, 950.0, Not Active, Not Active, Not Active, Not Active\n",
        "GPU-aaaa, 1965, 1965, 980.0, Active, Not Active, Not Active, Not Active\n",
        "garbage line\n",
    ]
    s = cs.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_clock_summary_without_samples_says_so():
    b = _bench()
    cs = b.ClockSampler("GPU-aaaa")
    cs.error = "no nvidia-smi"
    s = cs.summary()
    assert s["reasons"] == ["unsampled"] and s["sm_mhz"] is None

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


def test_torch_unpackers_match_the_layout_helper():
    """bench.py's torch unpackers (used by its fp64 quality evaluation) read
    the packed layout exactly as the tests' numpy helper does."""
    import numpy as np
    import torch

    from tests.layout import unpack_codes, unpack_signs
    b = _bench()
    rng = np.random.default_rng(0)
    for d, w in ((128, 1), (128, 2), (96, 3), (64, 3), (32, 4), (1536, 3)):
        raw = rng.integers(0, 256, size=(7, w * d // 8), dtype=np.uint8)
        got = b.unpack_codes_t(torch, torch.from_numpy(raw), d, w).numpy()
        assert np.array_equal(got, unpack_codes(raw, d, w))
    raw = rng.integers(0, 256, size=(5, 16), dtype=np.uint8)
    assert np.array_equal(b.unpack_signs_t(torch, torch.from_numpy(raw), 128).numpy(), unpack_signs(raw, 128))


def test_traffic_is_null_once_the_source_changes(monkeypatch):
    b = _bench()
    digest = b._source_digest("tq_api.cu")
    monkeypatch.setattr(b, "TRAFFIC", {"k@w": ("tq_api.cu", digest, 123, "small case"),
                                       "old@w": ("tq_api.cu", "0" * 16, 456, "small case")})
    assert b.traffic_for("k", "w") == (123, "small case")
    assert b.traffic_for("k", "other") == (None, None)  # a capture holds for its own workload only
    assert b.traffic_for("k") == (None, None)
    assert b.traffic_for("old", "w") == (None, None)
    assert b.traffic_for("missing", "w") == (None, None)


def test_device_errors_checks_every_quantizer():
    """After a timed region the bench asks the library for each quantizer's
    error word; an error (a kernel that gave up a bounded wait) fails the run."""
    b = _bench()
    seen = []

    class FakeTq:
        @staticmethod
        def tq_sync_check(q):
            seen.append(q)
            if q == "bad":
                raise RuntimeError("a kernel gave up a bounded wait")

    b.device_errors(FakeTq, "qa", "qb")
    assert seen == ["qa", "qb"]
    import pytest
    with pytest.raises(RuntimeError):
        b.device_errors(FakeTq, "qa", "bad", "qc")


def test_phases_off_run_the_work_without_events():
    """Timed steps run with the phase recorder switched off: the work still
    runs, and no CUDA event is created (so none sits between two kernels)."""
    b = _bench()

    class NoCuda:
        class cuda:
            @staticmethod
            def Event(**kw):
                raise AssertionError("no event while phases are off")

    ph = b.Phases(NoCuda, None)
    ph.enabled = False
    ran = []
    ph("encode", lambda: ran.append(1))
    assert ran == [1] and ph.ev == {}

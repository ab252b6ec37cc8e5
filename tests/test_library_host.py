"""CPU-only checks of libtq: it loads, exports every entry point of
include/tq.h, validates arguments, and its host-built tables (codebook,
rotation, QJL projection) agree with the oracle's independent construction."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import tq_oracle as o
from tests.layout import code_bit_position

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def tq():
    from online_vector_quantization_tq_b200 import build
    build.build()
    import online_vector_quantization_tq_b200 as pkg
    pkg.lib()
    return pkg


def test_exports_every_declared_symbol(tq):
    hdr = open(os.path.join(ROOT, "include", "tq.h")).read()
    names = set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", hdr))
    assert len(names) >= 15
    so = ctypes.CDLL(tq.binding.LIB_PATH)
    for name in sorted(names):
        assert hasattr(so, name), name


@pytest.mark.parametrize("d,b", [(128, 4), (128, 3), (96, 3), (32, 5), (1536, 4)])
def test_code_bytes(tq, d, b):
    """Packed bytes per vector = w*d/8 codes + m/8 sign bits + two fp32 norms
    (72 B for the kv shape d=128, b=4; 776 B for d=1536, b=4)."""
    q = tq.tq_codebook_host(d, b, seed=0)
    assert tq.lib().tq_code_bytes(q.handle) == (b - 1) * d // 8 + d // 8 + 8
    assert tq.lib().tq_code_bytes(q.handle) == q.code_bytes + q.sign_bytes + 8
    assert tq.lib().tq_code_bytes(None) == 0


def test_status_strings(tq):
    L = tq.lib()
    for code in range(7):
        assert L.tq_status_string(code)
    assert L.tq_status_string(99) == b"unknown status"


@pytest.mark.parametrize("d,b,rot", [(128, 3, "auto"), (128, 4, "auto"), (32, 5, "auto"), (64, 2, "auto"),
                                     (96, 3, "auto"), (256, 3, "haar"), (1536, 4, "auto")])
def test_host_tables_match_oracle(tq, d, b, rot):
    q = tq.tq_codebook_host(d, b, seed=0, rotation=rot)
    t = o.Tables(d, b, seed=0, rotation=rot)
    c, thr, mse = q.codebook()
    scale = np.max(np.abs(t.centroids))
    assert np.max(np.abs(c - t.centroids)) < 1e-12 * scale
    assert np.max(np.abs(thr - t.thresholds)) < 1e-12 * scale
    assert abs(mse - t.coord_mse) < 1e-12 * mse
    R, diag, S = q.tables()
    assert np.array_equal(S.view(np.float16).astype(np.float64), t.S)
    if q.rotation == "hadamard":
        for r, stream in enumerate((o.STREAM_D1, o.STREAM_D2, o.STREAM_D3)):
            assert np.array_equal(diag[r].astype(np.float64), o.rademacher(0, stream, d))
        # the dense product rounded once to fp32
        assert np.all(np.abs(R.astype(np.float64) - t.R) <= np.abs(t.R) * 2.0 ** -24 + 1e-15)
    else:
        # same fp32 matrix up to rare one-ulp differences from the two QR codes
        diff = R.astype(np.float64) - t.R
        assert np.max(np.abs(diff)) <= np.max(np.abs(t.R)) * 2.0 ** -23
        assert np.count_nonzero(diff) <= max(4, d * d // 100000)


def test_deterministic_in_seed(tq):
    a = tq.tq_codebook_host(128, 3, seed=7).tables()
    b = tq.tq_codebook_host(128, 3, seed=7).tables()
    c = tq.tq_codebook_host(128, 3, seed=8).tables()
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    assert not np.array_equal(a[2], c[2])


@pytest.mark.parametrize("args,code", [((100, 3), 2), ((128, 1), 1), ((128, 6), 1), ((0, 3), 1),
                                       ((4128, 3), 2)])
def test_codebook_argument_errors(tq, args, code):
    with pytest.raises(tq.TQError) as e:
        tq.tq_codebook_host(*args)
    assert e.value.code == code
    with pytest.raises(tq.TQError) as e:
        tq.tq_codebook_host(96, 3, rotation="hadamard")
    assert e.value.code == 2
    with pytest.raises(tq.TQError) as e:
        tq.tq_codebook_host(64, 3, m=32)
    assert e.value.code == 2


def test_device_calls_refuse_host_only_quantizer(tq):
    """No GPU needed: the check happens before any pointer is touched."""
    q = tq.tq_codebook_host(128, 3)
    L = tq.lib()
    fake = ctypes.c_void_p(0x1000)
    st = L.tq_encode(q.handle, fake, 0, 16, 128, None, 0, fake, fake, fake, 1, None)
    assert st == 2
    st = L.tq_encode(None, fake, 0, 16, 128, None, 0, fake, fake, fake, 1, None)
    assert st == 1
    assert L.tq_qjl_matrix(q.handle, fake, None) == 2  # unsupported: no device tables
    assert L.tq_qjl_matrix(None, fake, None) == 1
    assert L.tq_set_qjl_onthefly(None, 1) == 1
    assert L.tq_set_qjl_onthefly(q.handle, 1) == 0 and L.tq_set_qjl_onthefly(q.handle, 0) == 0


def test_layout_is_a_bijection():
    for w in (1, 2, 3, 4):
        pos = sorted(code_bit_position(w, i, b) for i in range(32) for b in range(w))
        assert pos == list(range(32 * w))


@pytest.mark.parametrize("d,b", [(128, 3), (64, 1), (128, 4), (96, 2)])
def test_mse_mode_tables_match_oracle(tq, d, b):
    """TurboQuant-MSE quantizer: all b bits to the codebook (w = b), no QJL
    rows (m = 0, no sign bytes), and the same Lloyd-Max fit as the oracle's
    MSE-mode tables."""
    q = tq.tq_codebook_mse_host(d, b, seed=0)
    t = o.Tables(d, b, seed=0, mode="mse")
    assert (q.w, q.m, q.sign_bytes, q.code_bytes) == (b, 0, 0, b * d // 8)
    assert tq.lib().tq_code_bytes(q.handle) == b * d // 8 + 8
    c, thr, mse = q.codebook()
    scale = np.max(np.abs(t.centroids))
    assert np.max(np.abs(c - t.centroids)) < 1e-12 * scale
    assert np.max(np.abs(thr - t.thresholds)) < 1e-12 * scale
    assert abs(mse - t.coord_mse) < 1e-12 * mse
    for bad in (0, 5):
        with pytest.raises(tq.TQError):
            tq.tq_codebook_mse_host(d, bad, seed=0)


def test_encoded_views_must_be_contiguous(tq):
    """The library reads packed rows back to back, so the binding refuses a
    strided view of encoded rows (it would be read as if contiguous)."""
    import torch
    enc = tq.binding.Encoded(torch.zeros(64, 48, dtype=torch.uint8), torch.zeros(64, 16, dtype=torch.uint8),
                             torch.zeros(64, 2))
    enc.check()
    tq.binding.Encoded(enc.codes[8:], enc.signs[8:], enc.norms[8:]).check()  # a row offset is fine
    with pytest.raises(ValueError):
        tq.binding.Encoded(enc.codes[::4], enc.signs[::4], enc.norms[::4]).check()


def test_split_score_refuses_bad_arguments_before_any_launch(tq):
    """tq_score_prepare / tq_score_prepared validate on the host: a missing or
    host-only quantizer, missing key arrays and a short workspace are refused
    without touching a pointer (no GPU needed)."""
    q = tq.tq_codebook_host(128, 4)
    L = tq.lib()
    fake = ctypes.c_void_p(0x1000)
    assert L.tq_score_prepare(None, fake, 2, 4, 128, None, fake, 1 << 20, None) == 1
    assert L.tq_score_prepare(q.handle, fake, 2, 4, 128, None, fake, 1 << 20, None) == 2
    assert L.tq_score_prepare(q.handle, fake, -1, 4, 128, None, fake, 1 << 20, None) == 1
    assert L.tq_score_prepared(None, 2, 4, fake, fake, fake, 16, fake, 0, fake, 1 << 20, None) == 1
    assert L.tq_score_prepared(q.handle, 2, 4, fake, fake, fake, 16, fake, 0, fake, 1 << 20, None) == 2
    assert L.tq_score_prepared(q.handle, 2, 4, fake, fake, fake, -5, fake, 0, fake, 1 << 20, None) == 1

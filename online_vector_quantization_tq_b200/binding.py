"""Thin ctypes binding of libtq (include/tq.h) for PyTorch tensors.

Argument marshalling only: every step of encode, query preparation, scoring
and top-k runs in the library's CUDA kernels.  Tensors are passed as raw
device pointers with the caller's current CUDA stream.  If the shared
library is missing this module raises at load time; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_F32, TQ_BF16 = 0, 1
ROTATIONS = {"auto": 0, "hadamard": 1, "haar": 2}
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration",
          3: "misaligned pointer or leading dimension", 4: "out of memory",
          5: "CUDA error", 6: "workspace missing or too small",
          7: "request exceeds the fixed internal scratch buffer",
          8: "a kernel gave up a bounded wait; the outputs of that call are not valid"}

_lib = None


class TQError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} (status {code})")
        self.code = code


class _Info(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("b", ctypes.c_int), ("w", ctypes.c_int), ("m", ctypes.c_int),
                ("rotation", ctypes.c_int), ("device", ctypes.c_int), ("seed", ctypes.c_uint64),
                ("code_bytes", ctypes.c_size_t), ("sign_bytes", ctypes.c_size_t),
                ("coord_mse", ctypes.c_double)]


def lib() -> ctypes.CDLL:
    """Load libtq.so from the package directory (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libtq.so not built at {LIB_PATH}; run "
                          "`python online_vector_quantization_tq_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, u64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint64, ctypes.c_size_t
    sigs = {
        "tq_status_string": (ctypes.c_char_p, [i32]),
        "tq_codebook": (i32, [i32, i32, i32, u64, i32, ctypes.POINTER(vp)]),
        "tq_codebook_host": (i32, [i32, i32, i32, u64, i32, ctypes.POINTER(vp)]),
        "tq_codebook_mse": (i32, [i32, i32, u64, i32, ctypes.POINTER(vp)]),
        "tq_codebook_mse_host": (i32, [i32, i32, u64, i32, ctypes.POINTER(vp)]),
        "tq_destroy": (None, [vp]),
        "tq_info": (i32, [vp, ctypes.POINTER(_Info)]),
        "tq_code_bytes": (sz, [vp]),
        "tq_set_qjl_onthefly": (i32, [vp, i32]),
        "tq_attend_workspace_bytes": (sz, [vp, i64, i64, i64]),
        "tq_attend": (i32, [vp, vp, i64, i64, i64, ctypes.c_float, vp, vp, i64, i64, i64, vp, i64, vp, sz, vp]),
        "tq_qjl_matrix": (i32, [vp, vp, vp]),
        "tq_codebook_get": (i32, [vp, vp, vp, vp]),
        "tq_tables_get": (i32, [vp, vp, vp, vp]),
        "tq_encode": (i32, [vp, vp, i32, i64, i64, vp, i64, vp, vp, vp, i64, vp]),
        "tq_encode_workspace_bytes": (sz, [vp, i64]),
        "tq_encode_ws": (i32, [vp, vp, i32, i64, i64, vp, i64, vp, vp, vp, i64, vp, sz, vp]),
        "tq_prepare_queries": (i32, [vp, vp, i64, i64, vp, i64, vp, vp, vp]),
        "tq_score_workspace_bytes": (sz, [vp, i64]),
        "tq_score": (i32, [vp, vp, i64, i64, i64, vp, vp, vp, vp, i64, vp, i32, vp, sz, vp]),
        "tq_score_prepare": (i32, [vp, vp, i64, i64, i64, vp, vp, sz, vp]),
        "tq_score_prepared": (i32, [vp, i64, i64, vp, vp, vp, i64, vp, i32, vp, sz, vp]),
        "tq_topk_workspace_bytes": (sz, [vp, i64, i64, i32]),
        "tq_topk": (i32, [vp, vp, i64, i64, vp, vp, vp, i64, i32, vp, vp, vp, sz, vp]),
        "tq_score_noalloc": (i32, [vp, vp, i64, i64, i64, vp, vp, vp, vp, i64, vp, i32, vp]),
        "tq_rerank": (i32, [vp, i64, i64, vp, i32, i64, i64, i32, vp, i32, i32, vp, vp, vp]),
        "tq_outlier_workspace_bytes": (sz, [i64, i32]),
        "tq_outlier_channels": (i32, [vp, i32, i64, i64, i32, i64, i32, vp, vp, vp, sz, vp]),
        "tq_sync_check": (i32, [vp, vp]),
        "tq_selftest_timeout": (i32, [vp, vp]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(fn: str, code: int):
    if code != 0:
        raise TQError(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype(x: torch.Tensor) -> int:
    if x.dtype == torch.float32:
        return TQ_F32
    if x.dtype == torch.bfloat16:
        return TQ_BF16
    raise TypeError(f"unsupported dtype {x.dtype}")


def _ld(x: torch.Tensor) -> int:
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit stride in the last dimension")
    return x.stride(0)


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


@dataclass
class Encoded:
    codes: torch.Tensor   # uint8 [n, code_bytes]
    signs: torch.Tensor   # uint8 [n, sign_bytes]
    norms: torch.Tensor   # float32 [n, 2]: ||x||, gamma

    def check(self):
        """The library reads and writes whole packed rows back to back: every
        array must be row-contiguous (a strided view would be read as if it
        were not)."""
        for name in ("codes", "signs", "norms"):
            t = getattr(self, name)
            if t.numel() and not t.is_contiguous():
                raise ValueError(f"Encoded.{name} must be contiguous (got strides {t.stride()})")
        return self


class Quantizer:
    """Owned tq_quantizer handle."""

    def __init__(self, handle: ctypes.c_void_p):
        self._h = handle
        info = _Info()
        _check("tq_info", lib().tq_info(self._h, ctypes.byref(info)))
        self.d, self.b, self.w, self.m = info.d, info.b, info.w, info.m
        self.rotation = {1: "hadamard", 2: "haar"}[info.rotation]
        self.device_index = info.device
        self.seed = info.seed
        self.code_bytes, self.sign_bytes = info.code_bytes, info.sign_bytes
        self.coord_mse = info.coord_mse

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h:
            lib().tq_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def codebook(self):
        import numpy as np
        L = 1 << self.w
        c = np.zeros(L)
        t = np.zeros(L - 1)
        mse = ctypes.c_double()
        _check("tq_codebook_get", lib().tq_codebook_get(
            self._h, c.ctypes.data_as(ctypes.c_void_p), t.ctypes.data_as(ctypes.c_void_p), ctypes.byref(mse)))
        return c, t, mse.value

    def tables(self):
        """(R fp32 [d,d], diagonal signs int8 [3,d] or None, S fp16 bits uint16 [m,d])."""
        import numpy as np
        r = np.zeros((self.d, self.d), dtype=np.float32)
        diag = np.zeros((3, self.d), dtype=np.int8)
        s = np.zeros((self.m, self.d), dtype=np.uint16)
        _check("tq_tables_get", lib().tq_tables_get(
            self._h, r.ctypes.data_as(ctypes.c_void_p), diag.ctypes.data_as(ctypes.c_void_p),
            s.ctypes.data_as(ctypes.c_void_p)))
        return r, (diag if self.rotation == "hadamard" else None), s

    def empty_encoded(self, n: int, device="cuda") -> Encoded:
        return Encoded(torch.empty((n, self.code_bytes), dtype=torch.uint8, device=device),
                       torch.empty((n, self.sign_bytes), dtype=torch.uint8, device=device),
                       torch.empty((n, 2), dtype=torch.float32, device=device))


def tq_codebook(d: int, b: int, m: int = 0, seed: int = 0, rotation: str = "auto") -> Quantizer:
    h = ctypes.c_void_p()
    _check("tq_codebook", lib().tq_codebook(d, b, m, seed, ROTATIONS[rotation], ctypes.byref(h)))
    return Quantizer(h)


def tq_codebook_host(d: int, b: int, m: int = 0, seed: int = 0, rotation: str = "auto") -> Quantizer:
    h = ctypes.c_void_p()
    _check("tq_codebook_host", lib().tq_codebook_host(d, b, m, seed, ROTATIONS[rotation], ctypes.byref(h)))
    return Quantizer(h)


def tq_codebook_mse(d: int, b: int, seed: int = 0, rotation: str = "auto") -> Quantizer:
    """TurboQuant-MSE quantizer: all b bits to the codebook, no QJL sign bits."""
    h = ctypes.c_void_p()
    _check("tq_codebook_mse", lib().tq_codebook_mse(d, b, seed, ROTATIONS[rotation], ctypes.byref(h)))
    return Quantizer(h)


def tq_codebook_mse_host(d: int, b: int, seed: int = 0, rotation: str = "auto") -> Quantizer:
    h = ctypes.c_void_p()
    _check("tq_codebook_mse_host", lib().tq_codebook_mse_host(d, b, seed, ROTATIONS[rotation], ctypes.byref(h)))
    return Quantizer(h)


def tq_encode(q: Quantizer, x: torch.Tensor, out: Encoded | None = None, chan: torch.Tensor | None = None,
              chan_rows: int = 0, out_stride: int = 1, workspace: torch.Tensor | None = None,
              stream=None) -> Encoded:
    n = x.shape[0]
    if out is None:
        out = q.empty_encoded(n, x.device)
    out.check()
    if chan is not None and chan.dtype != torch.int32:
        raise TypeError("chan must be int32")
    L = lib()
    args = (q.handle, _ptr(x), _dtype(x), n, _ld(x), _ptr(chan), chan_rows,
            _ptr(out.codes), _ptr(out.signs), _ptr(out.norms), out_stride)
    if workspace is None:
        ws = L.tq_encode_workspace_bytes(q.handle, n)
        if ws:
            workspace = _workspace(ws, x.device)
    if workspace is None:
        _check("tq_encode", L.tq_encode(*args, _stream(stream)))
    else:
        _check("tq_encode_ws", L.tq_encode_ws(*args, _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def tq_prepare_queries(q: Quantizer, y: torch.Tensor, ychan: torch.Tensor | None = None, ychan_rows: int = 0,
                       stream=None):
    nq = y.shape[0]
    ytil = torch.empty((nq, q.d), dtype=torch.float32, device=y.device)
    p = torch.empty((nq, q.m), dtype=torch.float32, device=y.device)
    _check("tq_prepare_queries", lib().tq_prepare_queries(
        q.handle, _ptr(y), nq, _ld(y), _ptr(ychan), ychan_rows, _ptr(ytil), _ptr(p), _stream(stream)))
    return ytil, p


def score_workspace(q: Quantizer, nq: int, device="cuda") -> torch.Tensor:
    return _workspace(lib().tq_score_workspace_bytes(q.handle, nq), device)


def tq_score(q: Quantizer, y: torch.Tensor, groups: int, G: int, enc: Encoded, keys_per_group: int,
             out: torch.Tensor | None = None, accumulate: bool = False, ychan: torch.Tensor | None = None,
             workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    enc.check()
    if out is None:
        out = torch.empty((groups * G, keys_per_group), dtype=torch.float32, device=y.device)
    if workspace is None:
        workspace = score_workspace(q, groups * G, y.device)
    _check("tq_score", lib().tq_score(
        q.handle, _ptr(y), groups, G, _ld(y), _ptr(ychan), _ptr(enc.codes), _ptr(enc.signs), _ptr(enc.norms),
        keys_per_group, _ptr(out), int(bool(accumulate)), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def tq_score_prepare(q: Quantizer, y: torch.Tensor, groups: int, G: int, workspace: torch.Tensor | None = None,
                     ychan: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Query half of tq_score: writes the prepared queries into `workspace`
    (allocated when None) and returns it, for tq_score_prepared."""
    if workspace is None:
        workspace = score_workspace(q, groups * G, y.device)
    _check("tq_score_prepare", lib().tq_score_prepare(
        q.handle, _ptr(y), groups, G, _ld(y), _ptr(ychan), _ptr(workspace), workspace.numel(), _stream(stream)))
    return workspace


def tq_score_prepared(q: Quantizer, groups: int, G: int, enc: Encoded, keys_per_group: int,
                      workspace: torch.Tensor, out: torch.Tensor | None = None, accumulate: bool = False,
                      stream=None) -> torch.Tensor:
    """Key half of tq_score against the queries tq_score_prepare wrote into
    `workspace`."""
    enc.check()
    if out is None:
        out = torch.empty((groups * G, keys_per_group), dtype=torch.float32, device=enc.codes.device)
    _check("tq_score_prepared", lib().tq_score_prepared(
        q.handle, groups, G, _ptr(enc.codes), _ptr(enc.signs), _ptr(enc.norms), keys_per_group, _ptr(out),
        int(bool(accumulate)), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def topk_workspace(q: Quantizer, nq: int, n: int, k: int, device="cuda") -> torch.Tensor:
    return _workspace(lib().tq_topk_workspace_bytes(q.handle, nq, n, k), device)


def tq_topk(q: Quantizer, y: torch.Tensor, enc: Encoded, k: int, n: int | None = None,
            workspace: torch.Tensor | None = None, out=None, stream=None):
    """(scores fp32 [nq, k], key indices int64 [nq, k]); `out` may give both."""
    nq = y.shape[0]
    enc.check()
    n = enc.codes.shape[0] if n is None else n
    if out is None:
        vals = torch.empty((nq, k), dtype=torch.float32, device=y.device)
        idx = torch.empty((nq, k), dtype=torch.int64, device=y.device)
    else:
        vals, idx = out
    if workspace is None:
        workspace = topk_workspace(q, nq, n, k, y.device)
    _check("tq_topk", lib().tq_topk(
        q.handle, _ptr(y), nq, _ld(y), _ptr(enc.codes), _ptr(enc.signs), _ptr(enc.norms), n, k,
        _ptr(vals), _ptr(idx), _ptr(workspace), workspace.numel(), _stream(stream)))
    return vals, idx


def tq_attend(qv: Quantizer, logits: torch.Tensor, groups: int, G: int, venc: Encoded, keys_per_group: int,
              scale: float, key_base: int = 0, nkeys: int | None = None, out: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Attention over a quantized KV cache: softmax(scale * logits) times the
    TurboQuant-MSE reconstructions of the values (venc, encoded by qv), one
    row of d floats per query (groups*G rows)."""
    venc.check()
    n = keys_per_group - key_base if nkeys is None else nkeys
    if out is None:
        out = torch.empty((groups * G, qv.d), dtype=torch.float32, device=logits.device)
    if workspace is None:
        workspace = _workspace(lib().tq_attend_workspace_bytes(qv.handle, groups, G, n), logits.device)
    _check("tq_attend", lib().tq_attend(
        qv.handle, _ptr(logits), _ld(logits), groups, G, float(scale), _ptr(venc.codes),
        _ptr(venc.norms), keys_per_group, key_base, n, _ptr(out), _ld(out), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return out


def tq_set_qjl_onthefly(q: Quantizer, enable: bool = True) -> None:
    """Generate the QJL matrix S from the seed inside the kernels that can
    (see include/tq.h) instead of reading the stored table."""
    _check("tq_set_qjl_onthefly", lib().tq_set_qjl_onthefly(q.handle, int(bool(enable))))


def tq_qjl_matrix(q: Quantizer, device="cuda", stream=None) -> torch.Tensor:
    """S (m x d fp16 bit patterns as int16, row-major) generated on the
    device from the quantizer seed."""
    out = torch.empty((q.m, q.d), dtype=torch.int16, device=device)
    _check("tq_qjl_matrix", lib().tq_qjl_matrix(q.handle, _ptr(out), _stream(stream)))
    return out


def tq_rerank(y: torch.Tensor, x: torch.Tensor, cand: torch.Tensor, k: int, out=None, stream=None):
    """Second stage of two-stage retrieval: exact <y, x> of every candidate
    key (cand: int64 [nq, kc], e.g. tq_topk's indices) against the raw rows
    x, and the k best per query: (scores fp32 [nq, k], keys int64 [nq, k])."""
    nq, kc = cand.shape
    if out is None:
        vals = torch.empty((nq, k), dtype=torch.float32, device=y.device)
        idx = torch.empty((nq, k), dtype=torch.int64, device=y.device)
    else:
        vals, idx = out
    if cand.dtype != torch.int64 or not cand.is_contiguous():
        raise TypeError("cand must be a contiguous int64 tensor")
    _check("tq_rerank", lib().tq_rerank(
        _ptr(y), nq, _ld(y), _ptr(x), _dtype(x), x.shape[0], _ld(x), x.shape[1], _ptr(cand), kc, k,
        _ptr(vals), _ptr(idx), _stream(stream)))
    return vals, idx


def tq_outlier_channels(x: torch.Tensor, groups: int, rows_per_group: int, count: int, stream=None):
    """Per group, the `count` highest-mean-square channels and the rest (both
    ascending int32 tensors on x's device)."""
    dim = x.shape[1]
    sel = torch.empty((groups, count), dtype=torch.int32, device=x.device)
    rest = torch.empty((groups, dim - count), dtype=torch.int32, device=x.device)
    ws = _workspace(lib().tq_outlier_workspace_bytes(groups, dim), x.device)
    _check("tq_outlier_channels", lib().tq_outlier_channels(
        _ptr(x), _dtype(x), groups, rows_per_group, dim, _ld(x), count, _ptr(sel), _ptr(rest),
        _ptr(ws), ws.numel(), _stream(stream)))
    return sel, rest


def tq_sync_check(q: "Quantizer", stream=None) -> None:
    """Synchronize `stream` and raise TQError (status 8) if a kernel of q gave
    up a bounded wait since the last check (its outputs are not valid)."""
    _check("tq_sync_check", lib().tq_sync_check(q.handle, _stream(stream)))


def tq_selftest_timeout(q: "Quantizer", stream=None) -> None:
    """Launch a kernel whose wait runs out (about 2 s): tests the failure path."""
    _check("tq_selftest_timeout", lib().tq_selftest_timeout(q.handle, _stream(stream)))

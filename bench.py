"""Throughput of the TurboQuant encode + score hot path on B200 GPUs.

Headline: one step = encode every key of one synthetic KV-cache layer (8 KV
heads x 131072 keys, head_dim 128, bf16, b = 4 bits) and score every key
against its 4 query heads (32 query heads, fp32 logits).  value = keys
through the whole step per second, summed over ranks (weak scaling: every
rank runs its own layer; the path shards by key with no collective).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]
                  [--workload all|kv|tiny|kv_mixed|decode|ann] [--queries Q]

With the default --workload all, rank 0 of a one-GPU run also times the
other four workloads (tiny, kv_mixed, decode, ann) and two variants (kv_mse:
the kv layer with TurboQuant-MSE keys; kv_mixed_2p5: the 2.5-bit outlier
split) and adds one record per workload to the headline line under
"configs": per-phase CUDA-event times,
the roofline of each phase's dominant kernel, quality figures of the encode
(code decisions and QJL sign bits against an fp64 evaluation, the raw sign
flip rate of a single-pass fp16 / bf16 projection), the scorer's worst error
against an fp64 evaluation, recall@10 (ann) and the oracle's CPU rate on a
bounded sample.  --workload NAME prints that workload's record alone.

Timing: CUDA events on the launching stream; barrier + synchronize around the
K timed steps; max over ranks.  L2 (126 MB): the kv workloads encode into one
of two code buffers per step and score the buffer written one step earlier,
so between the write and the read of a code buffer more than 330 MB of other
traffic (the 256 MiB key read, the other buffer) passes through L2; decode
(604 MB of codes) and ann (6 GB of keys) are larger than L2; tiny (2.3 MB)
is L2-resident by size and is launch-latency bound.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "keys scored/s and vectors encoded/s (1 B200), as % of HBM roofline"
CSRC = os.path.join(ROOT, "online_vector_quantization_tq_b200", "csrc")

# DRAM bytes (read + write) per launch counted by ncu for a kernel on one
# workload ("kernel@workload"), with the SHA-256 (first 16 hex digits) of the
# source file it was built from and of every header of the library, at the
# time of the capture.  A figure is reported only for that workload and while
# those sources are unchanged; otherwise the roofline's traffic is null.
TRAFFIC = {
    # kernel@workload: (source file, digest, bytes per launch, the capture)
    "k_encode_tc2@kv": ("tq_encode_tc.cu", "9831e14a2c4ee1a7", 326491392, "kv workload, launch 4, ncu --set full"),
    "k_score_tc@kv": ("tq_score_tc.cu", "29c8a83c49dff57f", 79304448, "kv workload, launch 4, ncu --set full"),
    "k_attend_split@decode_attend": ("tq_attend.cu", "8a7739e9493e3030", 616206848, "decode_attend workload, launch 3, ncu --set full"),
}


def _source_digest(fname: str) -> str:
    """Digest of a kernel's source file and of every header it may include."""
    h = hashlib.sha256()
    for name in [fname] + sorted(n for n in os.listdir(CSRC) if n.endswith((".h", ".cuh"))):
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload=None):
    ent = TRAFFIC.get(f"{kernel}@{workload}") if workload else None
    if not ent:
        return None, None
    fname, digest, nbytes, where = ent
    try:
        if _source_digest(fname) != digest:
            return None, None
    except OSError:
        return None, None
    return nbytes, where


def peaks() -> dict:
    """HBM GB/s and dense bf16 TFLOP/s: the measured figures of this GPU pool
    when the measured-peaks file is present, else the recipe's fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "kind": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "kind": "fallback"}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region.

    Samples every GPU the driver shows and keeps the one whose UUID matches
    the CUDA device (or the only one, when just one is visible).  A reader
    thread collects the lines as they come, so the caller can keep the GPU
    under load until samples have arrived."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = (uuid or "").lower().replace("gpu-", "")
        self.proc = None
        self.lines = []
        self.error = None
        self.thread = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln)

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception as e:  # no nvidia-smi
            self.error = str(e)
            self.proc = None
        return self

    def count(self) -> int:
        return len(self.lines)

    def wait_first(self, timeout: float = 20.0):
        t_end = time.time() + timeout
        while self.proc is not None and not self.lines and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.05)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                _, err = self.proc.communicate(timeout=5)
                if not self.lines:
                    self.error = (err or "").strip()[:200]
            except Exception:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=5)

    def summary(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = [[x.strip() for x in ln.split(",")] for ln in self.lines if ln.strip()]
        lines = [ln for ln in lines if len(ln) >= 8]
        uuids = sorted({ln[0].lower().replace("gpu-", "") for ln in lines})
        if self.uuid in uuids:
            lines = [ln for ln in lines if ln[0].lower().replace("gpu-", "") == self.uuid]
        elif len(uuids) > 1:
            lines = [ln for ln in lines if ln[0].lower().replace("gpu-", "") == uuids[0]]
        sm, mx, reasons = [], None, set()
        for ln in lines:
            try:
                sm.append(float(ln[1]))
                mx = float(ln[2])
            except ValueError:
                continue
            for nm, v in zip(names, ln[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "error": self.error}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------- timing

class Phases:
    """CUDA events around named phases of a step, on one stream."""

    def __init__(self, torch, stream):
        self.torch, self.stream = torch, stream
        self.ev = {}
        self.enabled = True

    def __call__(self, name, fn):
        if not self.enabled:
            fn()
            return
        a = self.torch.cuda.Event(enable_timing=True)
        b = self.torch.cuda.Event(enable_timing=True)
        a.record(self.stream)
        fn()
        b.record(self.stream)
        self.ev.setdefault(name, []).append((a, b))

    def clear(self):
        self.ev.clear()

    def mean_ms(self):
        return {k: statistics.mean(a.elapsed_time(b) for a, b in v) for k, v in self.ev.items()}


def device_errors(tq, *qs):
    """Raise if a kernel of these quantizers recorded an error during the steps
    (a bounded wait that gave up): their results, and the time, would be void."""
    for q in qs:
        tq.tq_sync_check(q)


def timed_steps(torch, dev, stream, step, steps, warmup, phases=None, clock=None):
    """W untimed warm-up steps, then K timed steps bracketed by synchronize;
    returns ms per step (CUDA events on `stream`).  The timed steps run with
    `phases` off: an event between two kernels would stop the second from
    starting in the first one's tail.  With `phases`, K more steps then record
    the per-phase events."""
    if phases is not None:
        phases.enabled = False
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1) / steps
    if phases is not None:
        phases.enabled = True
        phases.clear()
        for _ in range(steps):
            step()
        torch.cuda.synchronize(dev)
    return ms


def roofline_hbm(algo_bytes, ms, peak, kernel, unit_note, workload=None):
    traffic, where = traffic_for(kernel, workload)
    achieved = algo_bytes / (ms * 1e-3) / 1e9
    r = {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": peak["hbm_gbs"],
         "peak_kind": peak["kind"], "unit": "GB/s", "frac": achieved / peak["hbm_gbs"],
         "frac_of_nominal_8TBps": achieved / 8000.0, "traffic": traffic,
         "algorithmic_bytes_per_launch": algo_bytes, "algorithmic_bytes": unit_note}
    if where:
        r["traffic_capture"] = where
    return r


def roofline_tensor(algo_flops, ms, peak, kernel, unit_note, workload=None):
    traffic, where = traffic_for(kernel, workload)
    achieved = algo_flops / (ms * 1e-3) / 1e12
    r = {"bound": "tensor", "kernel": kernel, "achieved": achieved, "peak": peak["bf16_tflops_sustained"],
         "peak_kind": peak["kind"] + " (bf16 dense, sustained)", "unit": "TFLOP/s",
         "frac": achieved / peak["bf16_tflops_sustained"], "traffic": traffic,
         "algorithmic_flops_per_launch": algo_flops, "algorithmic_flops": unit_note}
    if where:
        r["traffic_capture"] = where
    return r


# ---------------------------------------------------------------------------- quality (evaluation only)
# Figures of the encode and the scorer measured against an fp64 evaluation of
# the method's definitions with torch on the GPU (like the exact fp32 ground
# truth of recall@10, this is evaluation arithmetic, not the product path).

def _code_positions(w):
    from tests.layout import code_bit_position
    return [[code_bit_position(w, i, b) for b in range(w)] for i in range(32)]


def unpack_codes_t(torch, codes_u8, d, w):
    n = codes_u8.shape[0]
    words = codes_u8.contiguous().view(torch.int32).view(n, d // 32, w).to(torch.int64) & 0xFFFFFFFF
    pos = torch.tensor(_code_positions(w), device=codes_u8.device)  # [32, w]
    sel = words[:, :, pos // 32]  # [n, g, 32, w]
    bits = (sel >> (pos % 32)) & 1
    return (bits << torch.arange(w, device=codes_u8.device)).sum(-1).view(n, d)


def unpack_signs_t(torch, signs_u8, m):
    n = signs_u8.shape[0]
    words = signs_u8.contiguous().view(torch.int32).view(n, m // 32, 1).to(torch.int64) & 0xFFFFFFFF
    return ((words >> torch.arange(32, device=signs_u8.device)) & 1).view(n, m).bool()


def quantizer_tables_t(torch, q, dev):
    R, _, S16 = q.tables()
    c, thr, _ = q.codebook()
    return (torch.from_numpy(R.astype(np.float64)).to(dev),
            torch.from_numpy(S16.view(np.float16).astype(np.float64)).to(dev),
            torch.from_numpy(c).to(dev), torch.from_numpy(thr).to(dev))


def encode_quality(torch, q, tabs, x, codes_u8, signs_u8, eps=1e-6):
    """Code decisions and sign bits of the kernel against fp64 evaluation.

    x: [k, d] device keys (bf16 or fp32), codes/signs: the kernel's packed rows.
    Code decisions: u = R x / ||x|| in fp64; a kernel code differing from
    #{thresholds < u} must lie within eps of a threshold.  Signs: with the
    kernel's codes, r = u - c[code], z = S r in fp64; the kernel's bit must be
    [z >= 0] unless |z| < eps.  Raw single-pass flip rates: the sign of S r
    computed once in fp16 (r scaled by 2^10 as the kernel does) and once in
    bf16, each with fp32 accumulation (cuBLAS), against the fp64 sign."""
    R, S, c, thr = tabs
    d, m, w = q.d, q.m, q.w
    x64 = x.double()
    nrm = torch.linalg.norm(x64, dim=1, keepdim=True)
    u = torch.where(nrm > 0, x64 / torch.where(nrm > 0, nrm, 1.0), 0.0) @ R.T
    ref_codes = torch.searchsorted(thr, u.contiguous(), right=False)
    kc = unpack_codes_t(torch, codes_u8, d, w)
    cmis = kc != ref_codes
    um = u[cmis]  # distance to the nearest threshold, where the decisions differ
    dist_mis = torch.min((um.unsqueeze(-1) - thr).abs(), dim=-1).values if um.numel() else um
    r = u - c[kc]
    if m == 0:  # TurboQuant-MSE: codes only
        return {"keys": int(x.shape[0]), "code_decisions": int(cmis.numel()), "code_mismatch": int(cmis.sum()),
                "code_mismatch_beyond_eps": int((dist_mis >= eps).sum()),
                "exempt_fraction": int(cmis.sum()) / max(1, int(cmis.numel()))}
    z = r @ S.T
    ref_bits = z >= 0
    kb = unpack_signs_t(torch, signs_u8, m)
    smis = kb != ref_bits
    torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = False
    torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction = False
    rs = (r * 1024.0)
    z16 = (rs.half() @ S.half().T).float()
    zb = (rs.bfloat16() @ S.bfloat16().T).float()
    big = z.abs() >= eps
    out = {
        "keys": int(x.shape[0]),
        "code_decisions": int(cmis.numel()),
        "code_mismatch": int(cmis.sum()),
        "code_mismatch_beyond_eps": int((dist_mis >= eps).sum()),
        "sign_bits": int(smis.numel()),
        "sign_mismatch": int(smis.sum()),
        "sign_mismatch_beyond_eps": int((smis & big).sum()),
        "raw_fp16_single_pass_flip_rate": float(((z16 >= 0) != ref_bits).double().mean()),
        "raw_fp16_flips_beyond_eps": int((((z16 >= 0) != ref_bits) & big).sum()),
        "raw_bf16_single_pass_flip_rate": float(((zb >= 0) != ref_bits).double().mean()),
        "raw_bf16_flips_beyond_eps": int((((zb >= 0) != ref_bits) & big).sum()),
    }
    out["exempt_fraction"] = (out["code_mismatch"] + out["sign_mismatch"]) / (out["code_decisions"]
                                                                              + out["sign_bits"])
    out["shipped_flip_rate"] = out["sign_mismatch"] / max(1, out["sign_bits"])
    return out


def score_quality(torch, q, tabs, y, codes_u8, signs_u8, norms, logits):
    """Worst error of the kernel's logits against the estimator evaluated in
    fp64 on the same codes, signs and norms: plain relative and floored
    (|s - s64| / max(|s64|, ||x|| ||y|| / sqrt(d)))."""
    R, S, c, _ = tabs
    ytil = y.double() @ R.T
    p = ytil @ S.T
    chat = c[unpack_codes_t(torch, codes_u8, q.d, q.w)]
    xn, gam = norms[:, 0].double(), norms[:, 1].double()
    if q.m == 0:  # TurboQuant-MSE: the codebook term alone
        s64 = xn[None, :] * (ytil @ chat.T)
    else:
        sig = unpack_signs_t(torch, signs_u8, q.m).double() * 2.0 - 1.0
        s64 = xn[None, :] * (ytil @ chat.T + (p @ sig.T) * (gam[None, :] * math.sqrt(math.pi / 2.0) / q.m))
    err = (logits.double() - s64).abs()
    floor = torch.linalg.norm(y.double(), dim=1)[:, None] * xn[None, :] / math.sqrt(q.d)
    plain = err / s64.abs().clamp_min(1e-300)
    return {"pairs": int(err.numel()), "max_err_floored": float((err / torch.maximum(s64.abs(), floor)).max()),
            "max_err_plain_relative": float(plain.max()),
            "max_err_plain_relative_p999": float(torch.quantile(plain.flatten()[:1 << 24].float(), 0.999))}


# ---------------------------------------------------------------------------- oracle (CPU baseline only)

def _oracle_rate(fn, target_s, start, limit):
    """Run fn(n) with n growing x4 until it takes target_s/4 or hits limit."""
    n = start
    dt = fn(n)
    while dt < target_s / 4 and n < limit:
        n = min(limit, n * 4)
        dt = fn(n)
    return n, dt


def _oracle_kv_sample(n_keys, b=4):
    import workloads as wl
    from oracle import tq_oracle as o
    t = o.Tables(128, b, seed=0)
    x = wl.kv_head_keys(0, 131072)[:n_keys]
    y = wl.kv_queries()[:4]
    t0 = time.perf_counter()
    enc = o.encode(x, t)
    o.score(*o.prepare_query(y, t), enc, t)
    return time.perf_counter() - t0


def _blas_threads(n):
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=n)


def _cores_used():
    try:
        from threadpoolctl import threadpool_info
        return int(max((i.get("num_threads", 1) for i in threadpool_info()), default=1))
    except Exception:
        return 1


def cpu_baseline(target_s=6.0):
    """Oracle (fp64 numpy) encode + score rate of the kv workload's keys, on a
    bounded sample, all cores and one thread."""
    ncpu = os.cpu_count() or 1
    with _blas_threads(ncpu):
        cores = _cores_used()
        n, dt = _oracle_rate(_oracle_kv_sample, target_s, 4096, 131072)
    with _blas_threads(1):
        n1, dt1 = _oracle_rate(_oracle_kv_sample, target_s / 2, 1024, 32768)
    return {"value": n / dt, "unit": "keys/s", "cores": cores, "host_cpus": ncpu, "kind": "oracle",
            "single_thread": {"value": n1 / dt1, "unit": "keys/s", "cores": 1,
                              "sample": f"{n1} keys, {dt1:.1f} s"},
            "sample": f"oracle fp64 encode + score (4 query heads) of the first {n} keys of KV head 0 of the kv "
                      f"workload, {dt:.1f} s on {cores} BLAS threads"}


def oracle_rate_for(name):
    """All-core oracle rate on a bounded sample of one workload (a few s)."""
    import workloads as wl
    from oracle import tq_oracle as o
    with _blas_threads(os.cpu_count() or 1):
        cores = _cores_used()
        if name == "tiny":
            t = o.Tables(128, 3, seed=0)
            x, y = wl.tiny_keys(), wl.tiny_queries()
            t0 = time.perf_counter()
            enc = o.encode(x, t)
            o.topk(o.score(*o.prepare_query(y, t), enc, t), 10)
            dt = time.perf_counter() - t0
            return {"value": x.shape[0] / dt, "unit": "keys/s", "cores": cores, "kind": "oracle",
                    "sample": f"the whole workload: 4096 keys encoded + 16 queries top-10, {dt:.2f} s"}
        if name == "decode_attend":
            t, tv = o.Tables(128, 3, seed=0), o.Tables(128, 3, seed=0, mode="mse")
            n = 8192
            x = wl.decode_group_keys(0, 32768)[:n]
            v = wl.decode_group_values(0, 32768)[:n]
            y = wl.decode_queries(1)
            t0 = time.perf_counter()
            enc, venc = o.encode(x, t), o.encode(v, tv)
            o.attend(o.score(*o.prepare_query(y, t), enc, t), 1.0 / math.sqrt(128), venc, tv)
            dt = time.perf_counter() - t0
            return {"value": n / dt, "unit": "keys/s", "cores": cores, "kind": "oracle",
                    "sample": f"{n} keys and values of cache 0 encoded, scored by its 4 query heads and attended, "
                              f"{dt:.2f} s"}
        if name == "kv_otf":
            t = o.Tables(128, 4, seed=0)
            n = 32768
            x = wl.kv_head_keys(0, 131072)[:n]
            y = wl.kv_queries()[:4]
            t0 = time.perf_counter()
            enc = o.encode(x, t)
            o.score(*o.prepare_query(y, t), enc, t)
            dt = time.perf_counter() - t0
            return {"value": n / dt, "unit": "keys/s", "cores": cores, "kind": "oracle",
                    "sample": f"{n} keys of KV head 0 encoded + scored by 4 query heads, {dt:.2f} s (the oracle "
                              "builds S once per quantizer either way)"}
        if name == "kv_mse":
            t = o.Tables(128, 3, seed=0, mode="mse")
            n = 32768
            x = wl.kv_head_keys(0, 131072)[:n]
            y = wl.kv_queries()[:4]
            t0 = time.perf_counter()
            enc = o.encode(x, t)
            o.score(*o.prepare_query(y, t), enc, t)
            dt = time.perf_counter() - t0
            return {"value": n / dt, "unit": "keys/s", "cores": cores, "kind": "oracle",
                    "sample": f"{n} keys of KV head 0 encoded (MSE mode) + scored by 4 query heads, {dt:.2f} s"}
        if name in ("kv_mixed", "kv_mixed_2p5"):
            (da, ba), (db, bb) = ((32, 5), (96, 3)) if name == "kv_mixed" else ((32, 4), (96, 2))
            ta, tb = o.Tables(da, ba, seed=0), o.Tables(db, bb, seed=0)
            n = 16384
            x = wl.kv_head_keys(0, 131072)[:n]
            y = wl.kv_queries()[:4]
            sel = o.outlier_channels(wl.kv_head_keys(0, 131072), 32)
            rest = np.setdiff1d(np.arange(128), sel)
            t0 = time.perf_counter()
            ea, eb = o.encode(x[:, sel], ta), o.encode(x[:, rest], tb)
            o.score(*o.prepare_query(y[:, sel], ta), ea, ta) + o.score(*o.prepare_query(y[:, rest], tb), eb, tb)
            dt = time.perf_counter() - t0
            return {"value": n / dt, "unit": "keys/s", "cores": cores, "kind": "oracle",
                    "sample": f"{n} keys of KV head 0 encoded (both parts) + scored by 4 query heads, {dt:.2f} s"}
        if name == "decode":
            t = o.Tables(128, 3, seed=0)
            x = wl.decode_group_keys(0, 32768)
            y = wl.decode_queries(1)
            t0 = time.perf_counter()
            enc = o.encode(x, t)
            o.score(*o.prepare_query(y, t), enc, t)
            dt = time.perf_counter() - t0
            return {"value": x.shape[0] / dt, "unit": "keys/s", "cores": cores, "kind": "oracle",
                    "sample": f"one (sequence, head) cache of 32768 keys encoded + scored by its 4 query heads, "
                              f"{dt:.2f} s"}
        if name == "ann":
            t = o.Tables(1536, 4, seed=0)
            n = 4096
            x = wl.ann_chunk(0)[:n]
            y = wl.ann_queries(16)
            t0 = time.perf_counter()
            enc = o.encode(x, t)
            o.topk(o.score(*o.prepare_query(y, t), enc, t), 10)
            dt = time.perf_counter() - t0
            return {"value": n / dt, "unit": "vectors/s", "cores": cores, "kind": "oracle",
                    "sample": f"{n} database vectors encoded + 16 queries scored and top-10 over them, {dt:.2f} s"}
    return None


# ---------------------------------------------------------------------------- inputs

def _pool():
    return cf.ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 4))


def kv_keys_host():
    import workloads as wl
    with _pool() as ex:
        heads = list(ex.map(lambda h: wl.kv_head_keys(h, 131072), range(8)))
    return np.stack(heads).reshape(-1, 128), wl.kv_queries()


# ---------------------------------------------------------------------------- headline: kv

def run_kv(args, rank, world, local, torch, tq, dev, stream, peak):
    import torch.distributed as dist
    groups, G, kpg, b = 8, 4, 131072, 4
    n = groups * kpg
    x_host_np, y_np = kv_keys_host()
    x_dev = torch.from_numpy(x_host_np).to(dev).to(torch.bfloat16)
    y_dev = torch.from_numpy(y_np).to(dev)
    q = tq.tq_codebook(128, b, seed=0)
    encs = [q.empty_encoded(n, dev) for _ in range(2)]
    logits = torch.empty((groups * G, kpg), dtype=torch.float32, device=dev)
    ws = tq.score_workspace(q, groups * G, dev)
    ph = Phases(torch, stream)
    it = [0]

    def step(record=True):
        i = it[0]
        it[0] += 1
        e_w, e_r = encs[i % 2], encs[(i + 1) % 2]
        if record:
            ph("encode", lambda: tq.tq_encode(q, x_dev, out=e_w, stream=stream))
            ph("score", lambda: tq.tq_score(q, y_dev, groups, G, e_r, kpg, out=logits, workspace=ws,
                                            stream=stream))
        else:
            tq.tq_encode(q, x_dev, out=e_w, stream=stream)
            tq.tq_score(q, y_dev, groups, G, e_r, kpg, out=logits, workspace=ws, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step(False)
    torch.cuda.synchronize(dev)
    w0 = time.perf_counter()
    for _ in range(4):
        step(False)
    torch.cuda.synchronize(dev)
    warm_ms = (time.perf_counter() - w0) * 250
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    props = torch.cuda.get_device_properties(dev)
    with ClockSampler(str(getattr(props, "uuid", ""))) as clk:
        # the same load before (until three samples came in, at most ~3 s)
        # and after the timed steps, so the 100 ms clock samples cover it
        clk.wait_first()
        n0, t_end = clk.count(), time.time() + 3.0
        while clk.count() < n0 + 3 and time.time() < t_end:
            for _ in range(max(1, int(50.0 / max(warm_ms, 1e-3)))):
                step(False)
            torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        # the timed steps carry no events between their kernels (an event there
        # would stop a kernel from starting in the previous one's tail)
        ms = timed_steps(torch, dev, stream, lambda: step(False), args.steps, 0, phases=None)
        device_errors(tq, q)
        if world > 1:
            dist.barrier()
        n1, t_end = clk.count(), time.time() + 1.0
        while clk.count() < n1 + 2 and time.time() < t_end:
            for _ in range(max(1, int(50.0 / max(warm_ms, 1e-3)))):
                step(False)
            torch.cuda.synchronize(dev)
    # per-phase times from as many more steps, with events between the phases
    ph.clear()
    for _ in range(args.steps):
        step(True)
    torch.cuda.synchronize(dev)
    pm = ph.mean_ms()
    enc_ms, score_ms = pm["encode"], pm["score"]
    if world > 1:
        t = torch.tensor([ms, enc_ms, score_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, enc_ms, score_ms = t.tolist()

    # end to end through the public API: pinned host keys in, logits out, every step
    x_pin = torch.from_numpy(x_host_np).to(torch.bfloat16).pin_memory()
    y_pin = torch.from_numpy(y_np).pin_memory()
    out_pin = torch.empty((groups * G, kpg), dtype=torch.float32).pin_memory()
    x_stage = torch.empty_like(x_dev)
    y_stage = torch.empty_like(y_dev)

    def e2e_step():
        x_stage.copy_(x_pin, non_blocking=True)
        y_stage.copy_(y_pin, non_blocking=True)
        tq.tq_encode(q, x_stage, out=encs[0], stream=stream)
        tq.tq_score(q, y_stage, groups, G, encs[0], kpg, out=logits, workspace=ws, stream=stream)
        out_pin.copy_(logits, non_blocking=True)

    if world > 1:
        dist.barrier()
    e2e_ms = timed_steps(torch, dev, stream, e2e_step, args.steps, max(1, args.warmup))
    device_errors(tq, q)
    if world > 1:
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = t.item()
        dist.barrier()

    enc_bytes_key = 128 * 2 + q.code_bytes + q.sign_bytes + 8
    score_bytes_key = q.code_bytes + q.sign_bytes + 8 + 4 * G
    line = {
        "metric": METRIC,
        "value": world * n / (ms * 1e-3),
        "unit": "keys/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 keys, fp32 arithmetic and logits",
        "data": "synthetic",
        "config": {"workload": "kv: 8 KV heads x 131072 keys, head_dim 128, bf16 N(0,1) with 4 channels "
                               "per head x10; 32 query heads (group 4); b=4; all fp32 logits",
                   "keys_per_step_per_gpu": n, "parallelism": f"dp{world} (independent layers, no collective)",
                   "l2": "no flush: keys (256 MiB) exceed L2; two code buffers, each step scores the codes "
                         "encoded one step earlier (>330 MB of other traffic in between)",
                   "step": "tq_encode (the keys), tq_score (the 32 queries against the keys encoded one "
                           "step earlier), on one stream"},
        "encode_vectors_per_s": world * n / (enc_ms * 1e-3),
        "score_keys_per_s": world * n / (score_ms * 1e-3),
        "score_logits_per_s": world * n * G / (score_ms * 1e-3),
        "encode_ms": enc_ms,
        "score_ms": score_ms,
        "roofline": roofline_hbm(n * enc_bytes_key, enc_ms, peak, "k_encode_tc2",
                                 f"{enc_bytes_key} B/key (256 in, 48 codes + 16 signs + 8 norms out) x {n} keys",
                                 workload="kv"),
        "score_roofline": dict(roofline_hbm(n * score_bytes_key, score_ms, peak, "k_score_tc",
                                            f"{score_bytes_key} B/key (72 in, 4 logits x 4 B out) x {n} keys",
                                            workload="kv"),
                               note="phase time: the fused query preparation kernel + the scorer (which starts "
                                    "during the preparation: programmatic dependent launch)"),
        "e2e": {"value": world * n / (e2e_ms * 1e-3), "unit": "keys/s",
                "h2d_bytes_per_step": x_pin.numel() * 2 + y_pin.numel() * 4,
                "d2h_bytes_per_step": out_pin.numel() * 4},
        "gpu_launches": args.steps * LAUNCHES_PER_STEP,
        "clocks": clk.summary(),
    }
    quality = None
    if rank == 0 and world == 1 and args.quality:
        tabs = quantizer_tables_t(torch, q, dev)
        rows = torch.arange(0, n, 16, device=dev)  # 65536 keys, every head
        e = encs[0]
        quality = {"encode": encode_quality(torch, q, tabs, x_dev[rows], e.codes[rows], e.signs[rows]),
                   "score": score_quality(torch, q, tabs, y_dev[:4], e.codes[:kpg:4], e.signs[:kpg:4],
                                          e.norms[:kpg:4], logits[:4, ::4]),
                   "sample": "encode: every 16th key (65536 keys); score: query heads 0-3 x every 4th key of "
                             "KV head 0"}
    return line, quality


# kernels of libtq launched per headline step: encode (1), the fused query
# preparation with the integer scorer's query operand (1), scoring (1)
LAUNCHES_PER_STEP = 3


# ---------------------------------------------------------------------------- the other workloads

def run_config(name, args, torch, tq, dev, stream, peak):
    """One workload's record: per-phase times, rooflines, quality figures."""
    import workloads as wl
    ph = Phases(torch, stream)
    rec = {}
    steps = args.steps if name != "ann" else min(args.steps, 10)
    if name == "tiny":
        x = torch.from_numpy(wl.tiny_keys()).to(dev)
        y = torch.from_numpy(wl.tiny_queries()).to(dev)
        q = tq.tq_codebook(128, 3, seed=0)
        enc = q.empty_encoded(x.shape[0], dev)
        ws = tq.topk_workspace(q, y.shape[0], x.shape[0], 10, dev)
        n = x.shape[0]

        def step():
            ph("encode", lambda: tq.tq_encode(q, x, out=enc, stream=stream))
            ph("topk", lambda: tq.tq_topk(q, y, enc, 10, workspace=ws, stream=stream))
        ms = timed_steps(torch, dev, stream, step, steps, max(3, args.warmup), ph)
        device_errors(tq, q)
        pm = ph.mean_ms()
        eb, sb = 512 + q.code_bytes + q.sign_bytes + 8, q.code_bytes + q.sign_bytes + 8
        rec = {"workload": "tiny: 4096 keys d=128 fp32 N(0,1), b=3, 16 queries, top-10",
               "value": n / (ms * 1e-3), "unit": "keys/s", "ms_per_step": ms, "phases_ms": pm,
               "bound": "launch latency (2.3 MB of data, L2-resident)",
               "roofline": {"encode": roofline_hbm(n * eb, pm["encode"], peak, "k_encode_fwht", f"{eb} B/key"),
                            "topk": roofline_hbm(n * sb, pm["topk"], peak, "k_score_tc", f"{sb} B/key")}}
        tabs = quantizer_tables_t(torch, q, dev)
        logits = tq.tq_score(q, y, 1, 16, enc, n)
        rec["quality"] = {"encode": encode_quality(torch, q, tabs, x, enc.codes, enc.signs),
                          "score": score_quality(torch, q, tabs, y, enc.codes, enc.signs, enc.norms, logits)}
    elif name in ("kv_mixed", "kv_mixed_2p5"):
        kpg, groups, G = 131072, 8, 4
        (da, ba), (db, bb) = ((32, 5), (96, 3)) if name == "kv_mixed" else ((32, 4), (96, 2))
        bits = (da * (ba) + db * bb) / 128.0
        xs, y_np = kv_keys_host()
        x = torch.from_numpy(xs).to(dev).to(torch.bfloat16)
        y = torch.from_numpy(y_np).to(dev)
        sel, rest = tq.tq_outlier_channels(x, groups, kpg, 32)
        qa, qb = tq.tq_codebook(da, ba, seed=0), tq.tq_codebook(db, bb, seed=0)
        n = x.shape[0]
        encs = [(qa.empty_encoded(n, dev), qb.empty_encoded(n, dev)) for _ in range(2)]
        out = torch.empty((groups * G, kpg), device=dev)
        wsa, wsb = tq.score_workspace(qa, groups * G, dev), tq.score_workspace(qb, groups * G, dev)
        wse = torch.empty(max(16, tq.lib().tq_encode_workspace_bytes(qb.handle, n)), dtype=torch.uint8,
                          device=dev)
        it = [0]
        pa, pb = f"encode_d{da}_b{ba}", f"encode_d{db}_b{bb}"

        def step():
            i = it[0]
            it[0] += 1
            (ea, eb), (ra, rb) = encs[i % 2], encs[(i + 1) % 2]
            ph(pa, lambda: tq.tq_encode(qa, x, out=ea, chan=sel, chan_rows=kpg, stream=stream))
            ph(pb, lambda: tq.tq_encode(qb, x, out=eb, chan=rest, chan_rows=kpg, workspace=wse, stream=stream))
            ph("score", lambda: (tq.tq_score(qa, y, groups, G, ra, kpg, out=out, ychan=sel, workspace=wsa,
                                             stream=stream),
                                 tq.tq_score(qb, y, groups, G, rb, kpg, out=out, accumulate=True, ychan=rest,
                                             workspace=wsb, stream=stream)))
        ms = timed_steps(torch, dev, stream, step, steps, max(3, args.warmup), ph)
        device_errors(tq, qa, qb)
        pm = ph.mean_ms()
        enc_ms = pm[pa] + pm[pb]
        key_b = qa.code_bytes + qa.sign_bytes + 8 + qb.code_bytes + qb.sign_bytes + 8
        rec = {"workload": f"{name}: kv tensors, per head the 32 highest-RMS channels at b={ba} (d=32, Hadamard) "
                           f"+ 96 at b={bb} (d=96, Haar), scores summed ({bits:g} bits per channel)",
               "value": n / (ms * 1e-3), "unit": "keys/s", "ms_per_step": ms, "phases_ms": pm,
               "encode_vectors_per_s": n / (enc_ms * 1e-3), "score_keys_per_s": n / (pm["score"] * 1e-3),
               "bytes_per_key": key_b,
               "l2": "two code buffers; each step scores the codes encoded one step earlier",
               "roofline": {"encode": roofline_hbm(n * (256 + key_b), enc_ms, peak, "k_encode_tcg",
                                                   f"{256 + key_b} B/key (256 in, {key_b} out), both parts"),
                            "score": roofline_hbm(n * (key_b + 16), pm["score"], peak, "k_score_tc",
                                                  f"{key_b + 16} B/key ({key_b} in, 16 logits out), both parts")}}
        ea, eb = encs[0]
        rows = torch.arange(0, kpg, 4, device=dev)  # 32768 keys of head 0
        xa = x[rows][:, sel[0].long()]
        xb = x[rows][:, rest[0].long()]
        tabs_a, tabs_b = quantizer_tables_t(torch, qa, dev), quantizer_tables_t(torch, qb, dev)
        rec["quality"] = {pa: encode_quality(torch, qa, tabs_a, xa, ea.codes[rows], ea.signs[rows]),
                          pb: encode_quality(torch, qb, tabs_b, xb, eb.codes[rows], eb.signs[rows]),
                          "sample": "every 4th key of KV head 0"}
    elif name == "kv_mse":
        groups, G, kpg, b = 8, 4, 131072, 3
        xs, y_np = kv_keys_host()
        x = torch.from_numpy(xs).to(dev).to(torch.bfloat16)
        y = torch.from_numpy(y_np).to(dev)
        q = tq.tq_codebook_mse(128, b, seed=0)
        n = x.shape[0]
        encs = [q.empty_encoded(n, dev) for _ in range(2)]
        logits = torch.empty((groups * G, kpg), dtype=torch.float32, device=dev)
        ws = tq.score_workspace(q, groups * G, dev)
        it = [0]

        def step():
            i = it[0]
            it[0] += 1
            ph("encode", lambda: tq.tq_encode(q, x, out=encs[i % 2], stream=stream))
            ph("score", lambda: tq.tq_score(q, y, groups, G, encs[(i + 1) % 2], kpg, out=logits, workspace=ws,
                                            stream=stream))
        ms = timed_steps(torch, dev, stream, step, steps, max(3, args.warmup), ph)
        device_errors(tq, q)
        pm = ph.mean_ms()
        kb = q.code_bytes + 8
        rec = {"workload": "kv_mse: the kv workload with TurboQuant-MSE keys (b = 3 bits all to the codebook, no QJL "
                           "stage), 32 query heads, all fp32 logits",
               "value": n / (ms * 1e-3), "unit": "keys/s", "ms_per_step": ms, "phases_ms": pm,
               "encode_vectors_per_s": n / (pm["encode"] * 1e-3), "score_keys_per_s": n / (pm["score"] * 1e-3),
               "bytes_per_key": kb,
               "l2": "two code buffers; each step scores the codes encoded one step earlier",
               "roofline": {"encode": roofline_hbm(n * (256 + kb), pm["encode"], peak, "k_encode_tc2",
                                                   f"{256 + kb} B/key (256 in, 48 codes + 8 norms out)"),
                            "score": roofline_hbm(n * (kb + 16), pm["score"], peak, "k_score_tc",
                                                  f"{kb + 16} B/key ({kb} in, 16 logits out)")}}
        tabs = quantizer_tables_t(torch, q, dev)
        rows = torch.arange(0, n, 16, device=dev)
        e = encs[0]
        sc = tq.tq_score(q, y[:4], 1, 4, tq.binding.Encoded(e.codes[:kpg:4].contiguous(),
                                                              e.signs[:kpg:4].contiguous(),
                                                              e.norms[:kpg:4].contiguous()), kpg // 4)
        rec["quality"] = {"encode": encode_quality(torch, q, tabs, x[rows], e.codes[rows], e.signs[rows]),
                          "score": score_quality(torch, q, tabs, y[:4], e.codes[:kpg:4], e.signs[:kpg:4],
                                                 e.norms[:kpg:4], sc),
                          "inner_product_gain_1_minus_dD": 1.0 - 128 * q.coord_mse,
                          "sample": "encode: every 16th key; score: query heads 0-3 x every 4th key of KV head 0"}
    elif name == "kv_otf":
        groups, G, kpg = 8, 4, 131072
        xs, y_np = kv_keys_host()
        x = torch.from_numpy(xs).to(dev).to(torch.bfloat16)
        y = torch.from_numpy(y_np).to(dev)
        q = tq.tq_codebook(128, 4, seed=0)
        n = x.shape[0]
        ref = tq.tq_encode(q, x[:65536])  # stored S, for the bit-identity check
        tq.tq_set_qjl_onthefly(q, True)
        encs = [q.empty_encoded(n, dev) for _ in range(2)]
        logits = torch.empty((groups * G, kpg), dtype=torch.float32, device=dev)
        ws = tq.score_workspace(q, groups * G, dev)
        it = [0]

        def step():
            i = it[0]
            it[0] += 1
            ph("encode", lambda: tq.tq_encode(q, x, out=encs[i % 2], stream=stream))
            ph("score", lambda: tq.tq_score(q, y, groups, G, encs[(i + 1) % 2], kpg, out=logits, workspace=ws,
                                            stream=stream))
        ms = timed_steps(torch, dev, stream, step, steps, max(3, args.warmup), ph)
        device_errors(tq, q)
        pm = ph.mean_ms()
        kb = q.code_bytes + q.sign_bytes + 8
        e = encs[0]
        same = bool(torch.equal(e.codes[:65536], ref.codes) and torch.equal(e.signs[:65536], ref.signs)
                    and torch.equal(e.norms[:65536], ref.norms))
        rec = {"workload": "kv_otf: the kv workload with the QJL matrix S generated from the seed inside the "
                           "encode (per CTA, in shared memory) and the query preparation (per thread, its row) "
                           "instead of read from the stored table",
               "value": n / (ms * 1e-3), "unit": "keys/s", "ms_per_step": ms, "phases_ms": pm,
               "encode_vectors_per_s": n / (pm["encode"] * 1e-3), "score_keys_per_s": n / (pm["score"] * 1e-3),
               "bytes_per_key": kb,
               "l2": "two code buffers; each step scores the codes encoded one step earlier",
               "roofline": {"encode": roofline_hbm(n * (256 + kb), pm["encode"], peak, "k_encode_tc2",
                                                   f"{256 + kb} B/key (256 in, {kb} out)"),
                            "score": roofline_hbm(n * (kb + 16), pm["score"], peak, "k_score_tc",
                                                  f"{kb + 16} B/key ({kb} in, 16 logits out)")},
               "bit_identical_to_stored_S": {"keys": 65536, "codes_signs_norms_equal": same}}
        tq.tq_set_qjl_onthefly(q, False)
    elif name == "decode":
        groups, kpg, G = 256, 32768, 4
        q = tq.tq_codebook(128, 3, seed=0)
        cache = q.empty_encoded(groups * kpg, dev)
        new = torch.empty((groups, 128), dtype=torch.bfloat16, device=dev)
        with _pool() as ex:
            for g0 in range(0, groups, 32):  # 32 caches (512 MB of fp32 draws) at a time
                for g, xg in zip(range(g0, g0 + 32), ex.map(lambda g: wl.decode_group_keys(g, kpg),
                                                            range(g0, g0 + 32))):
                    xg = torch.from_numpy(xg).to(dev).to(torch.bfloat16)
                    part = tq.binding.Encoded(cache.codes[g * kpg:], cache.signs[g * kpg:],
                                              cache.norms[g * kpg:])
                    tq.tq_encode(q, xg[:kpg - 1], out=part, stream=stream)
                    new[g] = xg[kpg - 1]
        tail = tq.binding.Encoded(cache.codes[kpg - 1:], cache.signs[kpg - 1:], cache.norms[kpg - 1:])
        y = torch.from_numpy(wl.decode_queries(groups)).to(dev)
        out = torch.empty((groups * G, kpg), device=dev)
        ws = tq.score_workspace(q, groups * G, dev)
        n = groups * kpg

        def step():
            ph("append", lambda: tq.tq_encode(q, new, out=tail, out_stride=kpg, stream=stream))
            ph("score", lambda: tq.tq_score(q, y, groups, G, cache, kpg, out=out, workspace=ws, stream=stream))
        ms = timed_steps(torch, dev, stream, step, steps, max(3, args.warmup), ph)
        device_errors(tq, q)
        pm = ph.mean_ms()
        sb = q.code_bytes + q.sign_bytes + 8 + 4 * G
        rec = {"workload": "decode: 32 sequences x 8 KV heads = 256 caches x 32768 keys, d=128, bf16, b=3; step = "
                           "append 1 key per cache (256 keys) + score 4 query heads per cache against all its keys",
               "value": n / (ms * 1e-3), "unit": "keys/s", "ms_per_step": ms, "phases_ms": pm,
               "score_logits_per_s": n * G / (pm["score"] * 1e-3),
               "l2": "604 MB of codes per score phase, larger than L2",
               "roofline": {"append": roofline_hbm(groups * (256 + sb - 4 * G), pm["append"], peak, "k_encode_tc2",
                                                   "312 B per appended key (latency-bound: 256 keys)"),
                            "score": roofline_hbm(n * sb, pm["score"], peak, "k_score_tc",
                                                  f"{sb} B/key (56 in, 16 logits out)")}}
        tabs = quantizer_tables_t(torch, q, dev)
        last = torch.arange(groups, device=dev) * kpg + (kpg - 1)
        rec["quality"] = {"append": encode_quality(torch, q, tabs, new, cache.codes[last], cache.signs[last]),
                          "score": score_quality(torch, q, tabs, y[:4], cache.codes[:kpg], cache.signs[:kpg],
                                                 cache.norms[:kpg], out[:4]),
                          "sample": "encode: the 256 appended keys; score: all logits of cache 0"}
    elif name == "decode_attend":
        groups, kpg, G, bv = 256, 32768, 4, 3
        q = tq.tq_codebook(128, 3, seed=0)
        qv = tq.tq_codebook_mse(128, bv, seed=0)
        cache = q.empty_encoded(groups * kpg, dev)
        vcache = qv.empty_encoded(groups * kpg, dev)
        with _pool() as ex:
            for g0 in range(0, groups, 16):
                keys = list(ex.map(lambda g: wl.decode_group_keys(g, kpg), range(g0, g0 + 16)))
                vals = list(ex.map(lambda g: wl.decode_group_values(g, kpg), range(g0, g0 + 16)))
                for g, xg, vg in zip(range(g0, g0 + 16), keys, vals):
                    part = tq.binding.Encoded(cache.codes[g * kpg:], cache.signs[g * kpg:], cache.norms[g * kpg:])
                    tq.tq_encode(q, torch.from_numpy(xg).to(dev).to(torch.bfloat16), out=part, stream=stream)
                    vpart = tq.binding.Encoded(vcache.codes[g * kpg:], vcache.signs[g * kpg:],
                                               vcache.norms[g * kpg:])
                    tq.tq_encode(qv, torch.from_numpy(vg).to(dev).to(torch.bfloat16), out=vpart, stream=stream)
        y = torch.from_numpy(wl.decode_queries(groups)).to(dev)
        logits = torch.empty((groups * G, kpg), device=dev)
        att = torch.empty((groups * G, 128), device=dev)
        ws = tq.score_workspace(q, groups * G, dev)
        wsa = tq.binding._workspace(tq.lib().tq_attend_workspace_bytes(qv.handle, groups, G, kpg), dev)
        scale = 1.0 / math.sqrt(128)
        n = groups * kpg

        def step():
            ph("score", lambda: tq.tq_score(q, y, groups, G, cache, kpg, out=logits, workspace=ws, stream=stream))
            ph("attend", lambda: tq.tq_attend(qv, logits, groups, G, vcache, kpg, scale, out=att, workspace=wsa,
                                              stream=stream))
        ms = timed_steps(torch, dev, stream, step, steps, max(3, args.warmup), ph)
        device_errors(tq, q, qv)
        pm = ph.mean_ms()
        sb = q.code_bytes + q.sign_bytes + 8 + 4 * G
        ab = 4 * G + qv.code_bytes + 8
        rec = {"workload": "decode_attend: the decode caches (256 x 32768 keys, d=128, keys b=3 inner-product mode) "
                           "with values in TurboQuant-MSE b=3; step = all logits of 4 query heads per cache (tq_score) "
                           "+ softmax(logits / sqrt(d)) times the dequantized values (tq_attend)",
               "value": n / (ms * 1e-3), "unit": "keys/s", "ms_per_step": ms, "phases_ms": pm,
               "attend_keys_per_s": n / (pm["attend"] * 1e-3),
               "l2": "1.9 GB of key and value codes per step, larger than L2",
               "roofline": {"score": roofline_hbm(n * sb, pm["score"], peak, "k_score_tc",
                                                  f"{sb} B/key (56 in, 16 logits out)"),
                            "attend": roofline_hbm(n * ab, pm["attend"], peak, "k_attend_split",
                                                   f"{ab} B/key (16 logits, {qv.code_bytes} value codes, "
                                                   "8 value norms; the second read of the logits hits L2)",
                                                   workload="decode_attend")}}
        # quality: group 0's outputs against an fp64 evaluation of the same definition
        R, _, c, _ = quantizer_tables_t(torch, qv, dev)
        codes0 = unpack_codes_t(torch, vcache.codes[:kpg], 128, qv.w)
        vhat = vcache.norms[:kpg, 0].double()[:, None] * (c[codes0] @ R)
        pr = torch.softmax(scale * logits[:G].double(), dim=1)
        ref = pr @ vhat
        floor = pr @ vcache.norms[:kpg, 0].double()
        err = (att[:G].double() - ref).abs() / floor[:, None]
        rec["quality"] = {"attend": {"max_err_over_sum_p_norm": float(err.max()),
                                     "bound_2^-10": 2.0 ** -10,
                                     "sample": "the 4 query heads of cache 0, every output coordinate"}}
    elif name == "ann":
        n, d, nq = args.ann_rows, 1536, args.queries
        nch = (n + wl.ANN_CHUNK - 1) // wl.ANN_CHUNK
        x = torch.empty((n, d), device=dev)
        with _pool() as ex:
            futs = [ex.submit(wl.ann_chunk, c, n, d) for c in range(nch)]
            for c, fu in enumerate(futs):
                blk = fu.result()
                x[c * wl.ANN_CHUNK:c * wl.ANN_CHUNK + blk.shape[0]] = torch.from_numpy(blk).to(dev)
        y = torch.from_numpy(wl.ann_queries(1024, d)[:nq]).to(dev)
        q = tq.tq_codebook(d, 4, seed=0)
        enc = q.empty_encoded(n, dev)
        wse = torch.empty(max(16, tq.lib().tq_encode_workspace_bytes(q.handle, n)), dtype=torch.uint8, device=dev)
        ws = tq.topk_workspace(q, nq, n, 10, dev)
        vals = torch.empty((nq, 10), device=dev)
        idx = torch.empty((nq, 10), dtype=torch.int64, device=dev)

        def step():
            ph("encode", lambda: tq.tq_encode(q, x, out=enc, workspace=wse, stream=stream))
            ph("topk", lambda: tq.tq_topk(q, y, enc, 10, workspace=ws, out=(vals, idx), stream=stream))
        ms = timed_steps(torch, dev, stream, step, steps, max(3, args.warmup), ph)
        device_errors(tq, q)
        pm = ph.mean_ms()
        enc_flops = 2.0 * n * d * (d + d)
        topk_flops = 2.0 * nq * n * (d + d)
        rec = {"workload": f"ann: {n:,} x 1536 fp32 (std i^-0.5, L2-normalised), Haar rotation, b=4; {nq} queries, "
                           "top-10 by estimated inner product",
               "value": n / (ms * 1e-3), "unit": "vectors/s", "ms_per_step": ms, "phases_ms": pm,
               "encode_vectors_per_s": n / (pm["encode"] * 1e-3),
               "query_latency_ms_per_1024_queries": pm["topk"] * 1024 / nq,
               "l2": "6.1 GB of keys, larger than L2",
               "roofline": {"encode": roofline_tensor(enc_flops, pm["encode"], peak, "k_dense_gemm",
                                                      "2 d (d + m) flop per vector: rotation and QJL projection"),
                            "encode_hbm": roofline_hbm(n * (4 * d + 776), pm["encode"], peak, "k_dense_gemm",
                                                       "6920 B/vector (HBM is not the bound)"),
                            "topk": roofline_tensor(topk_flops, pm["topk"], peak, "k_dscore_gemm",
                                                    "2 (d + m) flop per (query, key) pair")}}
        torch.backends.cuda.matmul.allow_tf32 = False
        truth = []
        for q0 in range(0, nq, 128):  # exact fp32 inner products, evaluation only
            truth.append(torch.topk(y[q0:q0 + 128] @ x.T, 10, dim=1).indices)
        truth = torch.cat(truth)
        hits = sum(len(set(a) & set(b)) for a, b in zip(idx.cpu().tolist(), truth.cpu().tolist()))
        rec["recall_at_10_vs_exact_fp32"] = hits / (10.0 * nq)
        # two-stage retrieval: the quantized top-16, then exact re-scoring of those 16
        ws16 = tq.topk_workspace(q, nq, n, 16, dev)
        v16 = torch.empty((nq, 16), device=dev)
        i16 = torch.empty((nq, 16), dtype=torch.int64, device=dev)
        v2 = torch.empty((nq, 10), device=dev)
        i2 = torch.empty((nq, 10), dtype=torch.int64, device=dev)
        ph2 = Phases(torch, stream)

        def two_stage():
            ph2("topk16", lambda: tq.tq_topk(q, y, enc, 16, workspace=ws16, out=(v16, i16), stream=stream))
            ph2("rerank", lambda: tq.tq_rerank(y, x, i16, 10, out=(v2, i2), stream=stream))
        timed_steps(torch, dev, stream, two_stage, min(steps, 5), 2, ph2)
        hits2 = sum(len(set(a) & set(b)) for a, b in zip(i2.cpu().tolist(), truth.cpu().tolist()))
        rec["two_stage"] = {"first_stage_k": 16, "phases_ms": ph2.mean_ms(),
                            "recall_at_10_vs_exact_fp32": hits2 / (10.0 * nq),
                            "note": "exact fp32 inner products of the 16 quantized candidates against the raw "
                                    "vectors (TurboQuant article 4.2.2, second stage)"}
        tabs = quantizer_tables_t(torch, q, dev)
        rows = torch.arange(0, n, max(1, n // 16384), device=dev)[:16384]
        logits = tq.tq_score(q, y[:16], 1, 16, tq.binding.Encoded(enc.codes[rows], enc.signs[rows],
                                                                    enc.norms[rows]), rows.numel())
        rec["quality"] = {"encode": encode_quality(torch, q, tabs, x[rows], enc.codes[rows], enc.signs[rows]),
                          "score": score_quality(torch, q, tabs, y[:16], enc.codes[rows], enc.signs[rows],
                                                 enc.norms[rows], logits),
                          "sample": "16384 keys spread over the database; score: 16 queries against them"}
        del x
    else:
        raise SystemExit(f"unknown workload {name}")
    if args.oracle:
        rec["cpu_baseline"] = oracle_rate_for(name)
    torch.cuda.synchronize(dev)
    return rec


# ---------------------------------------------------------------------------- drivers

def run_tq(args, rank, world, local):
    import torch
    import torch.distributed as dist

    import online_vector_quantization_tq_b200 as tq

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    stream = torch.cuda.current_stream(dev)
    peak = peaks()
    if args.workload not in ("all", "kv"):
        if rank == 0:
            rec = run_config(args.workload, args, torch, tq, dev, stream, peak)
            print(json.dumps({"metric": METRIC, "workload": args.workload, "n_gpus": 1, "steps": args.steps,
                              "warmup": args.warmup, **rec}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return
    line, quality = run_kv(args, rank, world, local, torch, tq, dev, stream, peak)
    if rank == 0:
        line["peaks"] = peak
        if quality is not None:
            line["quality"] = quality
        if world == 1:
            line["cpu_baseline"] = cpu_baseline()
            if args.workload == "all":
                configs = {"kv": {"workload": line["config"]["workload"], "value": line["value"], "unit": "keys/s",
                                  "ms_per_step": line["ms_per_step"],
                                  "phases_ms": {"encode": line["encode_ms"], "score": line["score_ms"]},
                                  "roofline": {"encode": line["roofline"], "score": line["score_roofline"]},
                                  "quality": quality, "cpu_baseline": line["cpu_baseline"]}}
                for name in ("tiny", "kv_mixed", "decode", "ann", "kv_mse", "kv_mixed_2p5", "kv_otf", "decode_attend"):
                    configs[name] = run_config(name, args, torch, tq, dev, stream, peak)
                    torch.cuda.empty_cache()
                line["configs"] = configs
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_reference(args, rank, world):
    if rank != 0:
        return
    n = 32768
    for _ in range(args.warmup):
        _oracle_kv_sample(n)
    times = [_oracle_kv_sample(n) for _ in range(args.steps)]
    dt = sum(times) / len(times)
    v = n / dt
    line = {"metric": METRIC, "value": v, "unit": "keys/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": "kv: 8 KV heads x 131072 keys, head_dim 128, bf16 N(0,1) with 4 channels "
                                   "per head x10; 32 query heads (group 4); b=4; all fp32 logits",
                       "sample_keys_per_step": n},
            "cpu_baseline": {"value": v, "unit": "keys/s", "cores": _cores_used(), "host_cpus": os.cpu_count(),
                             "kind": "oracle",
                             "sample": f"oracle fp64 encode + score of {n} keys of KV head 0 per step"},
            "e2e": {"value": v, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
    ap.add_argument("--workload", choices=["all", "kv", "tiny", "kv_mixed", "decode", "ann", "kv_mse",
                                           "kv_mixed_2p5", "kv_otf", "decode_attend"], default="all")
    ap.add_argument("--queries", type=int, default=1024, help="ann workload: number of queries")
    ap.add_argument("--ann-rows", type=int, default=1_000_000,
                    help="ann workload: database vectors (1e6 is the workload; fewer for profiling captures)")
    ap.add_argument("--no-quality", dest="quality", action="store_false",
                    help="skip the fp64 evaluation of the encode and the scorer")
    ap.add_argument("--no-oracle", dest="oracle", action="store_false",
                    help="skip the per-workload CPU oracle rates")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_tq(args, rank, world, local)


if __name__ == "__main__":
    main()

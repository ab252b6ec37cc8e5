"""Throughput of the TurboQuant encode + score hot path on B200 GPUs.

One step = encode every key of one synthetic KV-cache layer (8 KV heads x
131072 keys, head_dim 128, bf16, b = 4 bits) and score every key against its
4 query heads (32 query heads, fp32 logits).  value = keys through the whole
step per second, summed over ranks (weak scaling: every rank runs its own
layer; the path shards by key with no collective).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]
                  [--workload kv|tiny|kv_mixed|decode|ann] [--queries Q]

The default (kv) is the headline line; the other workloads print a line with
per-phase times on one GPU.

Rank 0 prints one JSON line.  Timing: CUDA events on the launching stream,
barrier + synchronize around the K timed steps, max over ranks.  The keys
(256 MiB per rank) are larger than the 126 MB L2, so no explicit flush is
needed between steps.  --impl reference times the CPU oracle (fp64 numpy)
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
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
# DRAM bytes (read + write) of one launch on the kv workload, from the ncu
# captures summarised in profiles/encode_tc2_kv.md and profiles/score_tc_kv.md;
# set to None whenever the kernel changes after its capture.
ENCODE_TRAFFIC_BYTES = 324954624
SCORE_TRAFFIC_BYTES = 79161326


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _bf16_peak():
    """Dense bf16 TFLOP/s measured on this machine (burst), else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


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


# ---------------------------------------------------------------------------- workloads

def kv_layer_host(n_per_head=131072):
    import workloads as wl
    x = np.stack([wl.kv_head_keys(h, n_per_head) for h in range(8)]).reshape(-1, 128)
    return x, wl.kv_queries()


def run_tq(args, rank, world, local):
    import torch
    import torch.distributed as dist

    import online_vector_quantization_tq_b200 as tq

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    groups, G, kpg, b = 8, 4, 131072, 4
    n = groups * kpg
    x_host_np, y_np = kv_layer_host(kpg)
    x_dev = torch.from_numpy(x_host_np).to(dev).to(torch.bfloat16)
    y_dev = torch.from_numpy(y_np).to(dev)
    q = tq.tq_codebook(128, b, seed=0)
    enc = q.empty_encoded(n, dev)
    logits = torch.empty((groups * G, kpg), dtype=torch.float32, device=dev)
    ws = tq.score_workspace(q, groups * G, dev)
    stream = torch.cuda.current_stream(dev)

    ev = {}

    def step(record=None):
        if record is not None:
            a, b_, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            a.record(stream)
        tq.tq_encode(q, x_dev, out=enc, stream=stream)
        if record is not None:
            b_.record(stream)
        tq.tq_score(q, y_dev, groups, G, enc, kpg, out=logits, workspace=ws, stream=stream)
        if record is not None:
            c.record(stream)
            record.append((a, b_, c))

    w0 = torch.cuda.Event(enable_timing=True)
    w1 = torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    for _ in range(args.warmup):
        step()
    w1.record(stream)
    torch.cuda.synchronize(dev)
    warm_ms = w0.elapsed_time(w1) / max(1, args.warmup)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    props = torch.cuda.get_device_properties(dev)
    recs = []
    with ClockSampler(str(getattr(props, "uuid", ""))) as clk:
        # the same load before (until three samples came in, at most ~3 s)
        # and after the timed steps, so the 100 ms clock samples cover it
        clk.wait_first()
        n0, t_end = clk.count(), time.time() + 3.0
        while clk.count() < n0 + 3 and time.time() < t_end:
            for _ in range(max(1, int(0.05 / max(warm_ms * 1e-3, 1e-5)))):
                step()
            torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step(recs)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        n1, t_end = clk.count(), time.time() + 1.0
        while clk.count() < n1 + 2 and time.time() < t_end:
            for _ in range(max(1, int(0.05 / max(warm_ms * 1e-3, 1e-5)))):
                step()
            torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1) / args.steps
    enc_ms = statistics.mean(a.elapsed_time(b_) for a, b_, _ in recs)
    score_ms = statistics.mean(b_.elapsed_time(c) for _, b_, c in recs)
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
        tq.tq_encode(q, x_stage, out=enc, stream=stream)
        tq.tq_score(q, y_stage, groups, G, enc, kpg, out=logits, workspace=ws, stream=stream)
        out_pin.copy_(logits, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / args.steps
    if world > 1:
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = t.item()
        dist.barrier()

    if rank == 0:
        peak, peak_kind = _peaks()
        enc_bytes = n * (128 * 2 + q.code_bytes + q.sign_bytes + 8)
        score_bytes = n * (q.code_bytes + q.sign_bytes + 8 + 4 * G)
        achieved = enc_bytes / (enc_ms * 1e-3) / 1e9
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
                       "l2": "inputs (256 MiB keys per rank) larger than the 126 MB L2; no flush"},
            "encode_vectors_per_s": world * n / (enc_ms * 1e-3),
            "score_keys_per_s": world * n / (score_ms * 1e-3),
            "score_logits_per_s": world * n * G / (score_ms * 1e-3),
            "encode_ms": enc_ms,
            "score_ms": score_ms,
            "roofline": {"bound": "hbm", "kernel": "encode", "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": ENCODE_TRAFFIC_BYTES,
                         "algorithmic_bytes_per_launch": enc_bytes},
            "score_roofline": {"bound": "hbm", "achieved": score_bytes / (score_ms * 1e-3) / 1e9, "peak": peak,
                               "unit": "GB/s", "frac": score_bytes / (score_ms * 1e-3) / 1e9 / peak,
                               "traffic": SCORE_TRAFFIC_BYTES,
                               "note": "phase time: query preparation kernels + the scorer"},
            "e2e": {"value": world * n / (e2e_ms * 1e-3), "unit": "keys/s",
                    "h2d_bytes_per_step": x_pin.numel() * 2 + y_pin.numel() * 4,
                    "d2h_bytes_per_step": out_pin.numel() * 4},
            "gpu_launches": args.steps * LAUNCHES_PER_STEP,
            "clocks": clk.summary(),
        }
        if world == 1:
            line["cpu_baseline"] = cpu_baseline()
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_workload(args):
    """The other workloads on one GPU (tiny, kv_mixed, decode, ann).  Prints
    one JSON line with the step time, per-phase times and algorithmic GB/s."""
    import torch

    import online_vector_quantization_tq_b200 as tq
    import workloads as wl

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    phases = {}
    flops_ = {}

    def timed(name, fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        phases.setdefault(name, []).append((a, b))

    if args.workload == "tiny":
        x = torch.from_numpy(wl.tiny_keys()).to(dev)
        y = torch.from_numpy(wl.tiny_queries()).to(dev)
        q = tq.tq_codebook(128, 3, seed=0)
        enc = q.empty_encoded(x.shape[0], dev)
        ws = tq.topk_workspace(q, y.shape[0], x.shape[0], 10, dev)
        n_units, unit = x.shape[0], "keys/s"
        bytes_ = {"encode": x.shape[0] * (512 + q.code_bytes + q.sign_bytes + 8),
                  "topk": x.shape[0] * (q.code_bytes + q.sign_bytes + 8)}
        desc = "tiny: 4096 keys d=128 fp32 N(0,1), b=3, 16 queries, top-10"

        def step():
            timed("encode", lambda: tq.tq_encode(q, x, out=enc, stream=stream))
            timed("topk", lambda: tq.tq_topk(q, y, enc, 10, workspace=ws, stream=stream))
    elif args.workload == "kv_mixed":
        kpg, groups, G = 131072, 8, 4
        xs = np.stack([wl.kv_head_keys(h, kpg) for h in range(groups)]).reshape(-1, 128)
        x = torch.from_numpy(xs).to(dev).to(torch.bfloat16)
        y = torch.from_numpy(wl.kv_queries()).to(dev)
        sel, rest = tq.tq_outlier_channels(x, groups, kpg, 32)
        qa, qb = tq.tq_codebook(32, 5, seed=0), tq.tq_codebook(96, 3, seed=0)
        ea, eb = qa.empty_encoded(x.shape[0], dev), qb.empty_encoded(x.shape[0], dev)
        out = torch.empty((groups * G, kpg), device=dev)
        wsa, wsb = tq.score_workspace(qa, groups * G, dev), tq.score_workspace(qb, groups * G, dev)
        n_units, unit = x.shape[0], "keys/s"
        bytes_ = {"encode": x.shape[0] * (256 + 72), "score": x.shape[0] * (72 + 16)}
        desc = ("kv_mixed: kv tensors, per head 32 highest-RMS channels at b=5 (d=32) + 96 at b=3 (d=96, Haar), "
                "scores summed")

        def step():
            timed("encode", lambda: (tq.tq_encode(qa, x, out=ea, chan=sel, chan_rows=kpg, stream=stream),
                                     tq.tq_encode(qb, x, out=eb, chan=rest, chan_rows=kpg, stream=stream)))
            timed("score", lambda: (tq.tq_score(qa, y, groups, G, ea, kpg, out=out, ychan=sel, workspace=wsa,
                                                stream=stream),
                                    tq.tq_score(qb, y, groups, G, eb, kpg, out=out, accumulate=True, ychan=rest,
                                                workspace=wsb, stream=stream)))
    elif args.workload == "decode":
        groups, kpg, G = 256, 32768, 4
        q = tq.tq_codebook(128, 3, seed=0)
        cache = q.empty_encoded(groups * kpg, dev)
        for g in range(groups):
            xg = torch.from_numpy(wl.decode_group_keys(g, kpg)).to(dev).to(torch.bfloat16)
            tq.tq_encode(q, xg, out=tq.binding.Encoded(cache.codes[g * kpg:], cache.signs[g * kpg:],
                                                        cache.norms[g * kpg:]))
            if g == 0:
                new = torch.empty((groups, 128), dtype=torch.bfloat16, device=dev)
            new[g] = xg[kpg - 1]
        tail = tq.binding.Encoded(cache.codes[kpg - 1:], cache.signs[kpg - 1:], cache.norms[kpg - 1:])
        y = torch.from_numpy(wl.decode_queries(groups)).to(dev)
        out = torch.empty((groups * G, kpg), device=dev)
        ws = tq.score_workspace(q, groups * G, dev)
        n_units, unit = groups * kpg, "keys/s"
        bytes_ = {"append": groups * (256 + 56), "score": groups * kpg * (56 + 16)}
        desc = "decode: 256 caches x 32768 keys, d=128, b=3; step = append 256 keys + score 4 heads per cache"

        def step():
            timed("append", lambda: tq.tq_encode(q, new, out=tail, out_stride=kpg, stream=stream))
            timed("score", lambda: tq.tq_score(q, y, groups, G, cache, kpg, out=out, workspace=ws, stream=stream))
    elif args.workload == "ann":
        n, d, nq = args.ann_rows, 1536, args.queries
        x = torch.empty((n, d), device=dev)
        for c in range((n + wl.ANN_CHUNK - 1) // wl.ANN_CHUNK):
            blk = wl.ann_chunk(c, n, d)
            x[c * wl.ANN_CHUNK:c * wl.ANN_CHUNK + blk.shape[0]] = torch.from_numpy(blk).to(dev)
        y = torch.from_numpy(wl.ann_queries(1024, d)[:nq]).to(dev)
        q = tq.tq_codebook(d, 4, seed=0)
        enc = q.empty_encoded(n, dev)
        wse = torch.empty(max(1, tq.lib().tq_encode_workspace_bytes(q.handle, n)), dtype=torch.uint8, device=dev)
        ws = tq.topk_workspace(q, nq, n, 10, dev)
        n_units, unit = n, "vectors/s"
        bytes_ = {"encode": n * (4 * d + q.code_bytes + q.sign_bytes + 8),
                  "topk": n * (q.code_bytes + q.sign_bytes + 8)}
        # the rotation and the QJL projection, and one product per (query, key,
        # coordinate of [y~ | p]): the dense contractions of the step
        flops_ = {"encode": 2.0 * n * d * (d + d), "topk": 2.0 * nq * n * (d + d)}
        desc = f"ann: {n:,} x 1536 fp32 (std i^-0.5, L2-normalised), Haar, b=4; {nq} queries, top-10"

        def step():
            timed("encode", lambda: tq.tq_encode(q, x, out=enc, workspace=wse, stream=stream))
            timed("topk", lambda: tq.tq_topk(q, y, enc, 10, workspace=ws, stream=stream))
    else:
        raise SystemExit(f"unknown workload {args.workload}")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    phases.clear()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1) / args.steps
    peak, peak_kind = _peaks()
    bf16_peak = _bf16_peak()
    ph = {}
    for name, evs in phases.items():
        pm = statistics.mean(a.elapsed_time(b) for a, b in evs)
        gbs = bytes_[name] / (pm * 1e-3) / 1e9
        ph[name] = {"ms": pm, "algorithmic_GBps": gbs, "frac_of_measured_hbm": gbs / peak}
        if name in flops_:
            tf = flops_[name] / (pm * 1e-3) / 1e12
            ph[name].update({"algorithmic_TFLOPs": tf, "frac_of_measured_bf16": tf / bf16_peak})
    line = {"metric": METRIC, "value": n_units / (ms * 1e-3), "unit": unit, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "data": "synthetic", "config": {"workload": desc}, "phases": ph,
            "peak_hbm_GBps": peak, "peak_kind": peak_kind}
    print(json.dumps(line), flush=True)


# kernels of libtq launched per step: encode (1), query preparation with the
# integer scorer's query operand (1), scoring (1)
LAUNCHES_PER_STEP = 3


def _oracle_sample(n_keys):
    """Oracle encode + score of the first n_keys keys of KV head 0 against its
    4 query heads; returns seconds."""
    import workloads as wl
    from oracle import tq_oracle as o
    t = o.Tables(128, 4, seed=0)
    x = wl.kv_head_keys(0, 131072)[:n_keys]
    y = wl.kv_queries()[:4]
    t0 = time.perf_counter()
    enc = o.encode(x, t)
    o.score(*o.prepare_query(y, t), enc, t)
    return time.perf_counter() - t0


def _cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(target_s=10.0):
    n = 16384
    dt = _oracle_sample(n)
    while dt < target_s / 4 and n < 131072:
        n = min(131072, n * 4)
        dt = _oracle_sample(n)
    return {"value": n / dt, "unit": "keys/s", "cores": _cores(), "kind": "oracle",
            "sample": f"oracle fp64 encode + score of {n} keys of KV head 0 (4 query heads), "
                      f"{dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    n = 32768
    for _ in range(args.warmup):
        _oracle_sample(n)
    times = [_oracle_sample(n) for _ in range(args.steps)]
    dt = sum(times) / len(times)
    v = n / dt
    line = {"metric": METRIC, "value": v, "unit": "keys/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": "kv: 8 KV heads x 131072 keys, head_dim 128, bf16 N(0,1) with 4 channels "
                                   "per head x10; 32 query heads (group 4); b=4; all fp32 logits",
                       "sample_keys_per_step": n},
            "cpu_baseline": {"value": v, "unit": "keys/s", "cores": _cores(), "kind": "oracle",
                             "sample": f"oracle fp64 encode + score of {n} keys of KV head 0 per step"},
            "e2e": {"value": v, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
    ap.add_argument("--workload", choices=["kv", "tiny", "kv_mixed", "decode", "ann"], default="kv")
    ap.add_argument("--queries", type=int, default=1024, help="ann workload: number of queries")
    ap.add_argument("--ann-rows", type=int, default=1_000_000,
                    help="ann workload: database vectors (1e6 is the workload; fewer for profiling captures)")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.workload != "kv":
        if rank == 0:
            run_workload(args)
        return
    run_tq(args, rank, world, local)


if __name__ == "__main__":
    main()

"""Throughput of the TurboQuant encode + score hot path on B200 GPUs.

One step = encode every key of one synthetic KV-cache layer (8 KV heads x
131072 keys, head_dim 128, bf16, b = 4 bits) and score every key against its
4 query heads (32 query heads, fp32 logits).  value = keys through the whole
step per second, summed over ranks (weak scaling: every rank runs its own
layer; the path shards by key with no collective).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]
                  [--workload kv|tiny|decode]

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


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self):
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "samples": len(sm), "reasons": sorted(reasons)}


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

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    recs = []
    with ClockSampler(gpu_id) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step(recs)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
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
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak, "traffic": None,
                         "algorithmic_bytes_per_launch": enc_bytes},
            "score_roofline": {"bound": "hbm", "achieved": score_bytes / (score_ms * 1e-3) / 1e9, "peak": peak,
                               "unit": "GB/s", "frac": score_bytes / (score_ms * 1e-3) / 1e9 / peak},
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


# kernels of libtq launched per step: encode (1), query preparation (1), scoring (1)
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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
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

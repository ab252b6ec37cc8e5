"""Seeded synthetic inputs for the five workloads (tests and bench).

This module only draws input data.  It holds none of the quantizer's
arithmetic, so both the CUDA path's tests and the CPU oracle may use it.
Every array is regenerated bit-for-bit from (seed, chunk): rows are drawn in
fixed chunks from ``numpy.random.default_rng([seed, chunk])`` so that a test
can rebuild any sampled chunk without drawing the whole workload.

Workloads (shapes follow the TurboQuant pages' use cases; the KV shapes are
those of an 8B-class GQA model, the ANN shape is the d=1536 embedding set the
TurboQuant article's section 3.3 evaluates, which is not available here):

  tiny      d=128 fp32 N(0,1), 4096 keys, 16 queries
  kv        8 KV heads x 131072 keys, d=128, bf16 N(0,1) with 4 channels per
            head scaled x10; 32 query heads (4 per KV head), bf16 N(0,1)
  kv_mixed  the kv tensors again (scored by a 32-channel + 96-channel split)
  decode    32 sequences x 8 KV heads x 32768 keys, d=128, bf16 N(0,1); the
            last key of every (sequence, head) is the one a decode step
            appends; 4 query heads per KV head
  ann       1,000,000 x 1536 fp32: Gaussian with per-dimension std i^-0.5
            (i = 1..1536), each row L2-normalised; 1024 queries, same law
"""
from __future__ import annotations

from dataclasses import dataclass

import math

import numpy as np

CONFIG_INDEX = {"tiny": 0, "kv": 1, "kv_mixed": 2, "decode": 3, "ann": 4}
QUANTIZER_SEED = 0


def data_seed(name: str) -> int:
    return 1000 + CONFIG_INDEX[name]


def query_seed(name: str) -> int:
    return 2000 + CONFIG_INDEX[name]


def to_bf16_values(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), returned as
    float32 holding exactly those bf16 values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    lsb = (bits >> np.uint64(16)) & np.uint64(1)
    bits = (bits + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return bits.astype(np.uint32).view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-exact."""
    return (np.ascontiguousarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


@dataclass(frozen=True)
class Workload:
    name: str
    d: int
    b: int
    groups: int            # independent key sets (KV heads, or 1)
    keys_per_group: int
    queries_per_group: int
    dtype: str             # "f32" or "bf16"
    topk: int = 0          # 0: all logits are produced


WORKLOADS = {
    "tiny": Workload("tiny", 128, 3, 1, 4096, 16, "f32", topk=10),
    "kv": Workload("kv", 128, 4, 8, 131072, 4, "bf16"),
    "kv_mixed": Workload("kv_mixed", 128, 0, 8, 131072, 4, "bf16"),
    "decode": Workload("decode", 128, 3, 256, 32768, 4, "bf16"),
    "ann": Workload("ann", 1536, 4, 1, 1_000_000, 1024, "f32", topk=10),
}

# kv_mixed: per head, the 32 highest-RMS channels at 5 bits, the other 96 at 3
MIXED_SPLIT = ((32, 5), (96, 3))
KV_OUTLIERS_PER_HEAD = 4
KV_OUTLIER_SCALE = 10.0


# ------------------------------------------------------------------ tiny

def tiny_keys() -> np.ndarray:
    return np.random.default_rng([data_seed("tiny"), 0]).standard_normal((4096, 128)).astype(np.float32)


def tiny_queries() -> np.ndarray:
    return np.random.default_rng([query_seed("tiny"), 0]).standard_normal((16, 128)).astype(np.float32)


# ------------------------------------------------------------------ kv

def kv_outlier_channels(head: int, name: str = "kv") -> np.ndarray:
    rng = np.random.default_rng([data_seed(name), 1_000_000 + head])
    return np.sort(rng.choice(128, size=KV_OUTLIERS_PER_HEAD, replace=False))


def kv_head_keys(head: int, n: int = 131072, name: str = "kv") -> np.ndarray:
    """Keys of one KV head as bf16-exact float32 values, [n, 128].

    kv and kv_mixed share these tensors (kv_mixed is the same layer encoded
    with a different bit split), so both draw from the kv seed."""
    rng = np.random.default_rng([data_seed("kv"), head])
    x = rng.standard_normal((n, 128), dtype=np.float32)
    x[:, kv_outlier_channels(head, "kv")] *= np.float32(KV_OUTLIER_SCALE)
    return to_bf16_values(x)


def kv_queries(q_heads: int = 32) -> np.ndarray:
    """Query heads as bf16-exact float32 values, [32, 128]; query head q
    belongs to KV head q // 4."""
    rng = np.random.default_rng([query_seed("kv"), 0])
    return to_bf16_values(rng.standard_normal((q_heads, 128), dtype=np.float32))


# ------------------------------------------------------------------ decode

def decode_group_keys(group: int, n: int = 32768) -> np.ndarray:
    """Cache of one (sequence, KV head) pair, bf16-exact float32 [n, 128];
    group = sequence * 8 + head.  Row n-1 is the key the decode step appends."""
    rng = np.random.default_rng([data_seed("decode"), group])
    return to_bf16_values(rng.standard_normal((n, 128), dtype=np.float32))


def decode_group_values(group: int, n: int = 32768) -> np.ndarray:
    """Values of the same cache, bf16-exact float32 [n, 128]: N(0,1) rows
    times a per-row scale drawn log-uniformly from [1/4, 4]."""
    rng = np.random.default_rng([data_seed("decode"), group, 1])
    v = rng.standard_normal((n, 128), dtype=np.float32)
    v *= np.exp(rng.uniform(-math.log(4.0), math.log(4.0), (n, 1))).astype(np.float32)
    return to_bf16_values(v)


def decode_queries(groups: int = 256) -> np.ndarray:
    rng = np.random.default_rng([query_seed("decode"), 0])
    return to_bf16_values(rng.standard_normal((groups * 4, 128), dtype=np.float32))


# ------------------------------------------------------------------ ann

ANN_CHUNK = 65536


def ann_std(d: int = 1536) -> np.ndarray:
    return (np.arange(1, d + 1, dtype=np.float64) ** -0.5).astype(np.float32)


def _ann_rows(rng, n, d):
    x = rng.standard_normal((n, d), dtype=np.float32) * ann_std(d)
    x /= np.linalg.norm(x.astype(np.float64), axis=1, keepdims=True).astype(np.float32)
    return x


def ann_chunk(chunk: int, n_total: int = 1_000_000, d: int = 1536) -> np.ndarray:
    """Database rows [chunk*65536, min((chunk+1)*65536, n_total))."""
    lo = chunk * ANN_CHUNK
    n = min(ANN_CHUNK, n_total - lo)
    return _ann_rows(np.random.default_rng([data_seed("ann"), chunk]), n, d)


def ann_rows(rows: np.ndarray, n_total: int = 1_000_000, d: int = 1536) -> np.ndarray:
    """Selected database rows, rebuilt from their chunks."""
    rows = np.asarray(rows)
    out = np.empty((rows.size, d), dtype=np.float32)
    for c in np.unique(rows // ANN_CHUNK):
        sel = np.nonzero(rows // ANN_CHUNK == c)[0]
        out[sel] = ann_chunk(int(c), n_total, d)[rows[sel] - c * ANN_CHUNK]
    return out


def ann_queries(nq: int = 1024, d: int = 1536) -> np.ndarray:
    return _ann_rows(np.random.default_rng([query_seed("ann"), 0]), nq, d)

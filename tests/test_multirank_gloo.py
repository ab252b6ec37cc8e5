"""The N>1 path on CPU: two gloo ranks shard a database by rows, take local
top-k, all-gather and merge; the result must equal the single-process top-k
(including the tie order).  Also the max-over-ranks timing reduction."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from online_vector_quantization_tq_b200.sharding import (allgather_topk, max_over_ranks, merge_topk,
                                                          shard_range)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _reference_topk(scores, k):
    nq, n = scores.shape
    vals = np.empty((nq, k), dtype=scores.dtype)
    idx = np.empty((nq, k), dtype=np.int64)
    for q in range(nq):
        order = np.lexsort((np.arange(n), -scores[q]))[:k]
        vals[q], idx[q] = scores[q, order], order
    return vals, idx


def _worker(rank, world, port, scores, k, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        n = scores.shape[1]
        lo, hi = shard_range(n, rank, world)
        local = torch.from_numpy(scores[:, lo:hi])
        kk = min(k, hi - lo)
        ls, li = merge_topk(local, torch.arange(lo, hi).expand(local.shape[0], -1).contiguous(), kk)
        if kk < k:  # pad empty slots
            pad = k - kk
            ls = torch.cat([ls, torch.full((ls.shape[0], pad), -float("inf"), dtype=ls.dtype)], 1)
            li = torch.cat([li, torch.full((li.shape[0], pad), -1, dtype=li.dtype)], 1)
        gs, gi = allgather_topk(ls, li, k)
        t = max_over_ranks([float(rank), 10.0 - rank])
        out[rank] = (gs.numpy(), gi.numpy(), t)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n,k", [(1000, 10), (7, 5)])
def test_two_rank_topk_matches_single_process(n, k):
    rng = np.random.default_rng(n)
    scores = np.round(rng.standard_normal((6, n)), 1).astype(np.float32)  # many ties
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        ctx = mp.get_context("spawn")
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, scores, k, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    rv, ri = _reference_topk(scores, k)
    for r in range(world):
        gs, gi, t = res[r]
        assert np.array_equal(gi, ri) and np.array_equal(gs, rv)
        assert t == [1.0, 10.0]


def test_shard_range_covers_rows():
    for n in (0, 1, 5, 1000):
        for world in (1, 2, 3, 8):
            spans = [shard_range(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1

"""GPU parity: the CUDA path (called through the C ABI) against the fp64
oracle on the same seeded inputs, for the five workloads and the edge cases.
Rules (exemptions, tolerances) are in tests/parity.py."""
import math

import numpy as np
import pytest
import torch

import workloads as wl
from oracle import tq_oracle as o
from tests.parity import check_encode, check_scores, check_topk, score_errors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from online_vector_quantization_tq_b200 import build
    build.build()
    import online_vector_quantization_tq_b200 as pkg
    pkg.lib()
    return pkg


_TABLES = {}


def tables(d, b, rot="auto"):
    key = (d, b, rot)
    if key not in _TABLES:
        _TABLES[key] = o.Tables(d, b, seed=wl.QUANTIZER_SEED, rotation=rot)
    return _TABLES[key]


def tables_mse(d, b, rot="auto"):
    key = (d, b, rot, "mse")
    if key not in _TABLES:
        _TABLES[key] = o.Tables(d, b, seed=wl.QUANTIZER_SEED, rotation=rot, mode="mse")
    return _TABLES[key]


def host(enc, rows=None):
    sl = slice(None) if rows is None else rows
    return (enc.codes[sl].cpu().numpy(), enc.signs[sl].cpu().numpy(), enc.norms[sl].cpu().numpy())


def dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dtype)


# ------------------------------------------------------------------ tiny

def test_tiny_encode_score_topk(tq):
    x = wl.tiny_keys()
    y = wl.tiny_queries()
    t = tables(128, 3)
    q = tq.tq_codebook(128, 3, seed=wl.QUANTIZER_SEED)
    enc = tq.tq_encode(q, dev(x))
    rep = check_encode(*host(enc), x, t)
    ytil, p = o.prepare_query(y, t)
    s_ref = o.score(ytil, p, rep.ref, t)
    s = tq.tq_score(q, dev(y), 1, 16, enc, 4096).cpu().numpy()
    check_scores(s, s_ref, rep.ref["norm"], np.linalg.norm(y, axis=1), 128, rep.skip_rows)
    vals, idx = tq.tq_topk(q, dev(y), enc, 10)
    vals, idx = vals.cpu().numpy(), idx.cpu().numpy()
    check_topk(vals, idx, s_ref, rep.ref["norm"], np.linalg.norm(y, axis=1), 128, 10)
    # top-k scores are the scorer's own values, bit for bit
    assert np.array_equal(vals, np.take_along_axis(s, idx, axis=1))


def test_prepared_queries(tq):
    y = wl.tiny_queries()
    for d, b in ((128, 3), (96, 3), (32, 5)):
        t = tables(d, b)
        q = tq.tq_codebook(d, b, seed=0)
        yy = y[:, :d].copy()
        ytil, p = tq.tq_prepare_queries(q, dev(yy))
        rt, rp = o.prepare_query(yy, t)
        assert np.allclose(ytil.cpu().numpy(), rt, rtol=0, atol=2e-5 * np.abs(rt).max())
        assert np.allclose(p.cpu().numpy(), rp, rtol=0, atol=2e-5 * np.abs(rp).max())


# ------------------------------------------------------------------ kv (8B-class GQA layer)

def _kv_tensor(n=131072):
    return np.stack([wl.kv_head_keys(h, n) for h in range(8)])  # [8, n, 128] bf16-exact fp32


def test_kv_full(tq):
    n = 131072
    xs = _kv_tensor(n)
    y = wl.kv_queries()
    t = tables(128, 4)
    q = tq.tq_codebook(128, 4, seed=0)
    x_dev = dev(xs.reshape(-1, 128), torch.bfloat16)
    enc = tq.tq_encode(q, x_dev)
    out = tq.tq_score(q, dev(y), 8, 4, enc, n).cpu().numpy()
    worst, exempt = 0.0, 0
    for h in range(8):
        rows = slice(h * n, (h + 1) * n)
        rep = check_encode(*host(enc, rows), xs[h], t)
        exempt += rep.n_code_exempt + rep.n_sign_exempt
        yh = y[4 * h:4 * h + 4]
        s_ref = o.score(*o.prepare_query(yh, t), rep.ref, t)
        worst = max(worst, check_scores(out[4 * h:4 * h + 4], s_ref, rep.ref["norm"],
                                        np.linalg.norm(yh, axis=1), 128, rep.skip_rows))
    print(f"kv: exempt coordinates {exempt}, worst score error {worst:.2e}")


# ------------------------------------------------------------------ kv_mixed (3.5-bit split)

def test_kv_mixed_full(tq):
    n = 131072
    xs = _kv_tensor(n)
    y = wl.kv_queries()
    x_dev = dev(xs.reshape(-1, 128), torch.bfloat16)
    sel, rest = tq.tq_outlier_channels(x_dev, 8, n, 32)
    sel, rest = sel.cpu().numpy(), rest.cpu().numpy()
    for h in range(8):
        ref_sel = o.outlier_channels(xs[h], 32)
        assert np.array_equal(sel[h], ref_sel)
        assert np.array_equal(rest[h], np.setdiff1d(np.arange(128), ref_sel))
        assert set(wl.kv_outlier_channels(h)) <= set(ref_sel.tolist())
    (da, ba), (db, bb) = wl.MIXED_SPLIT
    qa, qb = tq.tq_codebook(da, ba, seed=0), tq.tq_codebook(db, bb, seed=0)
    ta, tb = tables(da, ba), tables(db, bb)
    sel_d, rest_d = dev(sel, torch.int32), dev(rest, torch.int32)
    ea = tq.tq_encode(qa, x_dev, chan=sel_d, chan_rows=n)
    eb = tq.tq_encode(qb, x_dev, chan=rest_d, chan_rows=n)
    y_dev = dev(y)
    out = tq.tq_score(qa, y_dev, 8, 4, ea, n, ychan=sel_d)
    tq.tq_score(qb, y_dev, 8, 4, eb, n, out=out, accumulate=True, ychan=rest_d)
    out = out.cpu().numpy()
    worst = 0.0
    for h in range(8):
        rows = slice(h * n, (h + 1) * n)
        ra = check_encode(*host(ea, rows), xs[h][:, sel[h]], ta)
        rb = check_encode(*host(eb, rows), xs[h][:, rest[h]], tb)
        yh = y[4 * h:4 * h + 4]
        s_ref = (o.score(*o.prepare_query(yh[:, sel[h]], ta), ra.ref, ta)
                 + o.score(*o.prepare_query(yh[:, rest[h]], tb), rb.ref, tb))
        worst = max(worst, check_scores(out[4 * h:4 * h + 4], s_ref, np.linalg.norm(xs[h], axis=1),
                                        np.linalg.norm(yh, axis=1), 128, ra.skip_rows | rb.skip_rows))
    print(f"kv_mixed: worst score error {worst:.2e}")


# ------------------------------------------------------------------ decode step

def test_decode_step_full_size(tq):
    groups, n = 256, 32768
    t = tables(128, 3)
    q = tq.tq_codebook(128, 3, seed=0)
    x = torch.empty((groups * n, 128), dtype=torch.bfloat16, device="cuda")
    for g in range(groups):
        x[g * n:(g + 1) * n] = dev(wl.decode_group_keys(g, n), torch.bfloat16)
    cache = q.empty_encoded(groups * n)
    # the cache: the first n-1 keys of every group, written group by group
    for g in range(groups):
        part = tq.binding.Encoded(cache.codes[g * n:], cache.signs[g * n:], cache.norms[g * n:])
        tq.tq_encode(q, x[g * n:g * n + n - 1], out=part)
    # the decode step: one new key per group appended in place (out_stride = n)
    new = x.view(groups, n, 128)[:, n - 1, :].contiguous()
    tail = tq.binding.Encoded(cache.codes[n - 1:], cache.signs[n - 1:], cache.norms[n - 1:])
    tq.tq_encode(q, new, out=tail, out_stride=n)
    y = wl.decode_queries(groups)
    out = tq.tq_score(q, dev(y), groups, 4, cache, n).cpu().numpy()
    # every appended key (the decode step's own encode, written with a stride)
    appended = np.stack([wl.decode_group_keys(g, n)[n - 1] for g in range(groups)])
    last = np.arange(groups) * n + (n - 1)
    check_encode(cache.codes[last].cpu().numpy(), cache.signs[last].cpu().numpy(),
                 cache.norms[last].cpu().numpy(), appended, t)
    # all logits of 33 groups spread over the batch (every 8th, and the last)
    worst = 0.0
    for g in list(range(0, groups, 8)) + [groups - 1]:
        xg = wl.decode_group_keys(g, n)
        rows = slice(g * n, (g + 1) * n)
        rep = check_encode(*host(cache, rows), xg, t)
        yg = y[4 * g:4 * g + 4]
        s_ref = o.score(*o.prepare_query(yg, t), rep.ref, t)
        worst = max(worst, check_scores(out[4 * g:4 * g + 4], s_ref, rep.ref["norm"], np.linalg.norm(yg, axis=1),
                                        128, rep.skip_rows))
    print(f"decode: worst score error {worst:.2e} over 33 groups")


# ------------------------------------------------------------------ ANN d=1536

def test_ann_full_size(tq):
    """The whole ANN workload: 1e6 x 1536 keys encoded on the GPU and checked
    row by row against the oracle; 16 queries scored against all 1e6 keys
    (every logit compared with the oracle's); the GPU top-10 against the
    oracle's top-10 over the full score rows; recall@10 against exact fp32."""
    n, d, nq = 1_000_000, 1536, 16
    t = tables(d, 4)
    q = tq.tq_codebook(d, 4, seed=0)
    nchunks = (n + wl.ANN_CHUNK - 1) // wl.ANN_CHUNK
    x = torch.empty((n, d), dtype=torch.float32, device="cuda")
    for c in range(nchunks):
        blk = wl.ann_chunk(c, n, d)
        x[c * wl.ANN_CHUNK:c * wl.ANN_CHUNK + blk.shape[0]] = dev(blk)
    enc = tq.tq_encode(q, x)
    y = wl.ann_queries(1024, d)[:nq]
    y_dev = dev(y)
    s_all = tq.tq_score(q, y_dev, 1, nq, enc, n).cpu().numpy()
    vals, idx = tq.tq_topk(q, y_dev, enc, 10)
    vals, idx = vals.cpu().numpy(), idx.cpu().numpy()
    exact = y_dev @ x.T
    truth = torch.topk(exact, 10, dim=1).indices.cpu().numpy()
    del exact, x
    codes, signs, norms = host(enc)
    ytil, p = o.prepare_query(y, t)
    s_ref = np.empty((nq, n))
    xnorm = np.empty(n)
    skip = np.zeros(n, dtype=bool)
    exempt = 0
    for c in range(nchunks):
        lo = c * wl.ANN_CHUNK
        blk = wl.ann_chunk(c, n, d)
        rows = slice(lo, lo + blk.shape[0])
        rep = check_encode(codes[rows], signs[rows], norms[rows], blk, t)
        exempt += rep.n_code_exempt + rep.n_sign_exempt
        s_ref[:, rows] = o.score(ytil, p, rep.ref, t)
        xnorm[rows] = rep.ref["norm"]
        skip[rows] = rep.skip_rows
    ynorm = np.linalg.norm(y, axis=1)
    worst = check_scores(s_all, s_ref, xnorm, ynorm, d, skip)
    check_topk(vals, idx, s_ref, xnorm, ynorm, d, 10, skip)
    # the top-k path returns the scorer's own logits of its keys
    assert np.array_equal(vals, np.take_along_axis(s_all, idx, axis=1))
    recall = np.mean([len(set(idx[i]) & set(truth[i])) / 10 for i in range(nq)])
    print(f"ann: exempt decisions {exempt}, keys skipped {int(skip.sum())}, worst score error {worst:.2e}, "
          f"recall@10 {recall:.3f}")
    assert recall >= 0.8


# ------------------------------------------------------------------ dense paths and edge cases

@pytest.mark.parametrize("d,b,rot", [(128, 4, "haar"), (256, 3, "hadamard"), (64, 2, "auto"), (32, 5, "auto")])
def test_other_shapes(tq, d, b, rot):
    rng = np.random.default_rng(d + b)
    x = rng.standard_normal((1000, d)).astype(np.float32)
    y = rng.standard_normal((5, d)).astype(np.float32)
    t = tables(d, b, rot)
    q = tq.tq_codebook(d, b, seed=0, rotation=rot)
    enc = tq.tq_encode(q, dev(x))
    rep = check_encode(*host(enc), x, t)
    s = tq.tq_score(q, dev(y), 1, 5, enc, 1000).cpu().numpy()
    check_scores(s, o.score(*o.prepare_query(y, t), rep.ref, t), rep.ref["norm"], np.linalg.norm(y, axis=1),
                 d, rep.skip_rows)


@pytest.mark.parametrize("d,b,rot", [(384, 3, "haar"), (512, 5, "hadamard"), (320, 4, "haar")])
def test_dense_tensor_core_batches(tq, d, b, rot):
    """Dense rotation on the tensor cores (fp16-piece GEMMs), forced through several
    workspace batches: 1000 rows in batches of 256 (a ragged last batch), a zero row,
    and a partial 256-column tile when d is not a multiple of 256."""
    rng = np.random.default_rng(d * 7 + b)
    n = 1000
    x = (rng.standard_normal((n, d)) * 3.0).astype(np.float32)
    x[17] = 0.0
    t = tables(d, b, rot)
    q = tq.tq_codebook(d, b, seed=0, rotation=rot)
    nbytes = tq.lib().tq_encode_workspace_bytes(q.handle, 256)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    enc = tq.tq_encode(q, dev(x), workspace=ws)
    rep = check_encode(*host(enc), x, t)
    assert enc.norms[17, 0].item() == 0.0 and enc.norms[17, 1].item() > 0.0
    # a workspace too small for one 128-row batch is refused
    with pytest.raises(tq.TQError) as e:
        tq.tq_encode(q, dev(x[:4]), workspace=torch.empty(4096, dtype=torch.uint8, device="cuda"))
    assert e.value.code == 6
    y = rng.standard_normal((3, d)).astype(np.float32)
    s = tq.tq_score(q, dev(y), 1, 3, enc, n).cpu().numpy()
    assert np.all(s[:, 17] == 0.0)  # the zero key scores 0 (its relative error is undefined)
    skip = rep.skip_rows.copy()
    skip[17] = True
    check_scores(s, o.score(*o.prepare_query(y, t), rep.ref, t), rep.ref["norm"], np.linalg.norm(y, axis=1),
                 d, skip)


def test_dense_score_many_queries(tq):
    """Scoring for d > 128 (tensor-core GEMM over decoded keys): 200 queries (two
    query tiles, the second ragged) against 3000 keys (ragged key tiles); logits
    against the oracle, and top-k equal to the sorted logits."""
    d, b, n, nq = 384, 3, 3000, 200
    rng = np.random.default_rng(11)
    x = rng.standard_normal((n, d)).astype(np.float32)
    y = rng.standard_normal((nq, d)).astype(np.float32)
    t = tables(d, b, "haar")
    q = tq.tq_codebook(d, b, seed=0, rotation="haar")
    enc = tq.tq_encode(q, dev(x))
    rep = check_encode(*host(enc), x, t)
    s = tq.tq_score(q, dev(y), 1, nq, enc, n)
    s_ref = o.score(*o.prepare_query(y, t), rep.ref, t)
    check_scores(s.cpu().numpy(), s_ref, rep.ref["norm"], np.linalg.norm(y, axis=1), d, rep.skip_rows)
    vals, idx = tq.tq_topk(q, dev(y), enc, 10)
    sv, si = torch.sort(s, dim=1, descending=True, stable=True)
    assert torch.equal(vals, sv[:, :10]) and torch.equal(idx, si[:, :10])
    check_topk(vals.cpu().numpy(), idx.cpu().numpy(), s_ref, rep.ref["norm"], np.linalg.norm(y, axis=1), d, 10)
    # grouped scoring: 4 groups of 50 queries, each against its own 750 keys
    sg = tq.tq_score(q, dev(y), 4, 50, enc, 750).cpu().numpy()
    for g in range(4):
        ref_g = s_ref[g * 50:(g + 1) * 50, g * 750:(g + 1) * 750]
        check_scores(sg[g * 50:(g + 1) * 50], ref_g, rep.ref["norm"][g * 750:(g + 1) * 750],
                     np.linalg.norm(y[g * 50:(g + 1) * 50], axis=1), d, rep.skip_rows[g * 750:(g + 1) * 750])


def test_dense_topk_fused_chunks_and_ties(tq):
    """Top-k for d > 128 with the selection inside the scoring GEMM (no logits
    in memory): 70000 keys (three 32768-key chunks, the last ragged), 5 and
    130 queries (one and two query tiles), k = 1, 10, 16 (fused) and 20 (the
    chunked path); keys 0-499 repeated at 40000-40499 so that equal scores
    must come out by ascending key index.  Equal to a stable sort of
    tq_score's logits, bit for bit."""
    d, b, n = 384, 4, 70000
    rng = np.random.default_rng(21)
    x = rng.standard_normal((n, d)).astype(np.float32)
    x[40000:40500] = x[:500]
    q = tq.tq_codebook(d, b, seed=0, rotation="haar")
    enc = tq.tq_encode(q, dev(x))
    for nq in (5, 130):
        y = dev(rng.standard_normal((nq, d)).astype(np.float32))
        y[0] = dev(x[7])  # a query whose best keys are the duplicated pair 7 / 40007
        s = tq.tq_score(q, y, 1, nq, enc, n)
        sv, si = torch.sort(s, dim=1, descending=True, stable=True)
        for k in (1, 10, 16, 20):
            vals, idx = tq.tq_topk(q, y, enc, k)
            assert torch.equal(vals, sv[:, :k]) and torch.equal(idx, si[:, :k]), (nq, k)
        vals, idx = tq.tq_topk(q, y, enc, 2)
        assert idx[0].tolist() == [7, 40007]


@pytest.mark.parametrize("G", [12, 48])
def test_score_many_heads_per_group(tq, G):
    """The integer scorer with many queries per group: G = 12 (two accumulators,
    two key buffers) and G = 48 (one accumulator and one MMA issuer), two groups
    of 1500 keys (a ragged last tile), and a top-k over 100 queries (batches of
    48, 48 and 4)."""
    d, b, kpg, groups = 128, 4, 1500, 2
    rng = np.random.default_rng(G)
    x = rng.standard_normal((groups * kpg, d)).astype(np.float32)
    y = rng.standard_normal((groups * G, d)).astype(np.float32)
    t = tables(d, b)
    q = tq.tq_codebook(d, b, seed=0)
    enc = tq.tq_encode(q, dev(x))
    rep = check_encode(*host(enc), x, t)
    s = tq.tq_score(q, dev(y), groups, G, enc, kpg).cpu().numpy()
    yt = o.prepare_query(y, t)
    for g in range(groups):
        rows = slice(g * G, (g + 1) * G)
        keys = slice(g * kpg, (g + 1) * kpg)
        ref = {k: v[keys] for k, v in rep.ref.items()}
        s_ref = o.score(yt[0][rows], yt[1][rows], ref, t)
        check_scores(s[rows], s_ref, ref["norm"], np.linalg.norm(y[rows], axis=1), d, rep.skip_rows[keys])
    yq = rng.standard_normal((100, d)).astype(np.float32)
    n = groups * kpg
    vals, idx = tq.tq_topk(q, dev(yq), enc, 10)
    # the same query batches through tq_score use the same kernel: identical logits
    s_all = torch.cat([tq.tq_score(q, dev(yq[b0:b0 + 48]), 1, len(yq[b0:b0 + 48]), enc, n)
                       for b0 in range(0, 100, 48)])
    sv, si = torch.sort(s_all, dim=1, descending=True, stable=True)
    assert torch.equal(vals, sv[:, :10]) and torch.equal(idx, si[:, :10])
    s_ref = o.score(*o.prepare_query(yq, t), rep.ref, t)
    check_topk(vals.cpu().numpy(), idx.cpu().numpy(), s_ref, rep.ref["norm"], np.linalg.norm(yq, axis=1), d, 10)


def test_edge_cases(tq):
    t = tables(128, 3)
    q = tq.tq_codebook(128, 3, seed=0)
    rng = np.random.default_rng(3)
    # ragged n, a zero row, bf16 with padded leading dimension
    x = rng.standard_normal((333, 128)).astype(np.float32)
    x[5] = 0.0
    xb = wl.to_bf16_values(x)
    pad = torch.zeros((333, 136), dtype=torch.bfloat16, device="cuda")
    pad[:, :128] = dev(xb, torch.bfloat16)
    enc = tq.tq_encode(q, pad[:, :128])
    rep = check_encode(*host(enc), xb, t)
    assert enc.norms[5, 0].item() == 0.0
    s = tq.tq_score(q, dev(xb[:3]), 1, 3, enc, 333).cpu().numpy()
    assert np.all(s[:, 5] == 0.0)
    # n = 1 and n = 0
    one = tq.tq_encode(q, dev(x[:1]))
    check_encode(*host(one), x[:1], t)
    empty = q.empty_encoded(0)
    tq.tq_encode(q, torch.empty((0, 128), device="cuda"), out=empty)
    # channel gather: a permutation of 160 input channels
    wide = rng.standard_normal((200, 160)).astype(np.float32)
    perm = rng.permutation(160)[:128].astype(np.int32)
    enc2 = tq.tq_encode(q, dev(wide), chan=dev(perm[None, :], torch.int32), chan_rows=200)
    check_encode(*host(enc2), wide[:, perm], t)
    # argument errors return a status and launch nothing
    xx = dev(x)
    with pytest.raises(tq.TQError) as e:
        tq.tq_encode(q, xx.view(-1)[1:].view(-1)[:128 * 100].view(100, 128))
    assert e.value.code == 3
    with pytest.raises(tq.TQError) as e:
        tq.tq_score(q, xx[:2], 1, 2, enc, 333, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.code == 6
    with pytest.raises(tq.TQError) as e:
        tq.tq_topk(q, xx[:2], enc, 65)
    assert e.value.code == 1
    # tq_encode allocates nothing: a quantizer that needs scratch (Haar) is
    # refused there and encoded through tq_encode_ws
    qh = tq.tq_codebook(96, 3, seed=0)
    eh = qh.empty_encoded(4)
    st = tq.lib().tq_encode(qh.handle, tq.binding._ptr(xx[:4, :96].contiguous()), 0, 4, 96, None, 0,
                            tq.binding._ptr(eh.codes), tq.binding._ptr(eh.signs), tq.binding._ptr(eh.norms), 1,
                            tq.binding._stream(None))
    assert st == 6
    torch.cuda.synchronize()


# ------------------------------------------------------------------ TurboQuant-MSE mode

def test_mse_mode_kv_full(tq):
    """TurboQuant-MSE (all b = 3 bits to the codebook, no QJL sign bits) on
    the whole kv workload: bf16 keys through the tensor-core encode, codes
    and norms against the oracle's MSE mode, and every logit of the 32 query
    heads against the oracle's ||x|| <y~, c[codes]>."""
    n = 131072
    xs = _kv_tensor(n)
    y = wl.kv_queries()
    t = tables_mse(128, 3)
    q = tq.tq_codebook_mse(128, 3, seed=0)
    assert q.sign_bytes == 0 and q.w == 3
    enc = tq.tq_encode(q, dev(xs.reshape(-1, 128), torch.bfloat16))
    assert enc.signs.numel() == 0
    out = tq.tq_score(q, dev(y), 8, 4, enc, n).cpu().numpy()
    worst = 0.0
    for h in range(8):
        rows = slice(h * n, (h + 1) * n)
        rep = check_encode(*host(enc, rows), xs[h], t)
        yh = y[4 * h:4 * h + 4]
        s_ref = o.score(*o.prepare_query(yh, t), rep.ref, t)
        worst = max(worst, check_scores(out[4 * h:4 * h + 4], s_ref, rep.ref["norm"],
                                        np.linalg.norm(yh, axis=1), 128, rep.skip_rows))
    print(f"kv MSE mode: worst score error {worst:.2e}")


@pytest.mark.parametrize("d,b", [(128, 2), (64, 4), (32, 1)])
def test_mse_mode_fp32_and_topk(tq, d, b):
    """MSE mode for fp32 keys (the CUDA-core Hadamard encode), ragged tiles,
    a zero key, top-k against the oracle and against the scorer's own
    logits."""
    rng = np.random.default_rng(d * 10 + b)
    x = rng.standard_normal((3001, d)).astype(np.float32)
    x[9] = 0.0
    y = rng.standard_normal((7, d)).astype(np.float32)
    t = tables_mse(d, b)
    q = tq.tq_codebook_mse(d, b, seed=0)
    enc = tq.tq_encode(q, dev(x))
    rep = check_encode(*host(enc), x, t)
    s = tq.tq_score(q, dev(y), 1, 7, enc, 3001)
    s_ref = o.score(*o.prepare_query(y, t), rep.ref, t)
    check_scores(s.cpu().numpy(), s_ref, rep.ref["norm"], np.linalg.norm(y, axis=1), d, rep.skip_rows)
    vals, idx = tq.tq_topk(q, dev(y), enc, 10)
    sv, si = torch.sort(s, dim=1, descending=True, stable=True)
    assert torch.equal(vals, sv[:, :10]) and torch.equal(idx, si[:, :10])
    check_topk(vals.cpu().numpy(), idx.cpu().numpy(), s_ref, rep.ref["norm"], np.linalg.norm(y, axis=1), d, 10,
               rep.skip_rows)
    # an MSE quantizer refuses what it does not support (a Haar rotation)
    with pytest.raises(tq.TQError) as e:
        qh = tq.tq_codebook_mse(96, 3, seed=0)
        tq.tq_encode(qh, dev(rng.standard_normal((10, 96)).astype(np.float32)),
                     workspace=torch.empty(1 << 20, dtype=torch.uint8, device="cuda"))
    assert e.value.code == 2


# ------------------------------------------------------------------ two-stage retrieval

def _check_rerank(vals, idx, ref_v, ref_i, y, x, k):
    """Exact inner products in fp32 against fp64: |s - s64| <= (d + 2) 2^-24
    sum |y_i x_i| (a bound for any summation order); keys equal to the
    oracle's except where two candidates' exact scores lie within twice that
    bound of each other."""
    d = x.shape[1]
    for q in range(y.shape[0]):
        bound = (d + 2) * 2.0 ** -24 * (np.abs(x.astype(np.float64)) @ np.abs(y[q].astype(np.float64)))
        ok = ref_i[q] >= 0
        assert np.array_equal(idx[q] >= 0, ok)
        got = idx[q][ok]
        assert np.all(np.abs(vals[q][ok] - ref_v[q][ok]) <= bound[got])
        for j in np.nonzero(idx[q] != ref_i[q])[0]:
            a, b = idx[q][j], ref_i[q][j]
            assert a >= 0 and b >= 0
            assert abs(ref_v[q][j] - float(x[a].astype(np.float64) @ y[q])) <= 2 * (bound[a] + bound[b])
        assert np.all(vals[q][~ok] == -np.inf)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_rerank_against_oracle(tq, dtype):
    """Second stage on seeded candidate lists (duplicates, empty slots -1 and
    out-of-range keys included; a row with fewer valid candidates than k),
    fp32 and bf16 raw vectors, against the oracle's exact re-scoring."""
    rng = np.random.default_rng(17)
    n, d, nq, kc, k = 6000, 384, 40, 96, 10
    x = rng.standard_normal((n, d)).astype(np.float32)
    if dtype == "bf16":
        x = wl.to_bf16_values(x)
    x[123] = x[45]  # an exact tie
    y = rng.standard_normal((nq, d)).astype(np.float32)
    cand = rng.integers(0, n, size=(nq, kc))
    cand[:, 5] = cand[:, 6]        # duplicates
    cand[0, :2] = (45, 123)
    y[0] = x[45]
    cand[1, :] = -1                # a row with three valid candidates
    cand[1, :3] = (7, 8, 9)
    cand[2, 10] = n + 5            # out of range: an empty slot
    xd = dev(x, torch.bfloat16 if dtype == "bf16" else torch.float32)
    vals, idx = tq.tq_rerank(dev(y), xd, dev(cand, torch.int64), k)
    vals, idx = vals.cpu().numpy(), idx.cpu().numpy()
    cand_ref = np.where(cand < n, cand, -1)
    ref_v, ref_i = o.rerank(y, x, cand_ref, k)
    _check_rerank(vals, idx, ref_v, ref_i, y, x, k)
    assert idx[0][:2].tolist() == [45, 123]
    assert idx[1][3:].tolist() == [-1] * (k - 3)


def test_two_stage_retrieval_recall(tq):
    """Two-stage retrieval on an ANN-shaped sample (d = 1536, the ANN
    workload's law, 200000 keys, 64 queries): quantized top-100, then exact
    re-scoring of those 100; recall@10 against exact fp32 inner products is
    at least the first stage's and reaches 0.97 or more."""
    n, d, nq = 200000, 1536, 64
    x = torch.empty((n, d), dtype=torch.float32, device="cuda")
    for c in range((n + wl.ANN_CHUNK - 1) // wl.ANN_CHUNK):
        blk = wl.ann_chunk(c, n, d)
        x[c * wl.ANN_CHUNK:c * wl.ANN_CHUNK + blk.shape[0]] = dev(blk)
    y = dev(wl.ann_queries(1024, d)[:nq])
    q = tq.tq_codebook(d, 4, seed=0)
    enc = tq.tq_encode(q, x)
    v1, i1 = tq.tq_topk(q, y, enc, 10)
    vk, ik = tq.tq_topk(q, y, enc, 64)
    v2, i2 = tq.tq_rerank(y, x, ik, 10)
    torch.backends.cuda.matmul.allow_tf32 = False
    truth = torch.topk(y @ x.T, 10, dim=1).indices.cpu().numpy()
    r1 = np.mean([len(set(a) & set(b)) / 10 for a, b in zip(i1.cpu().numpy(), truth)])
    r2 = np.mean([len(set(a) & set(b)) / 10 for a, b in zip(i2.cpu().numpy(), truth)])
    print(f"two-stage: recall@10 first stage {r1:.3f}, after re-scoring the top-64 {r2:.3f}")
    assert r2 >= r1 and r2 >= 0.97


@pytest.mark.parametrize("d,b,rot", [(96, 2, "haar"), (32, 4, "hadamard"), (64, 3, "hadamard"), (64, 3, "haar")])
def test_gathered_bf16_encode(tq, d, b, rot):
    """bf16 rows of 128 channels encoded through a per-group channel map (the
    outlier split's path): 1000 rows in groups of 300 (group boundaries
    inside tiles, a ragged last tile), a zero row, codes and signs against
    the oracle on the gathered channels, scores with the same map."""
    rng = np.random.default_rng(d * 3 + b)
    n, rows_per_group = 1000, 300
    groups = (n + rows_per_group - 1) // rows_per_group
    x = wl.to_bf16_values(rng.standard_normal((n, 128)).astype(np.float32) * rng.choice([1.0, 7.0], size=128))
    x[11] = 0.0
    chan = np.stack([np.sort(rng.permutation(128)[:d]) for _ in range(groups)]).astype(np.int32)
    xg = np.stack([x[r, chan[r // rows_per_group]] for r in range(n)])
    t = tables(d, b, rot)
    q = tq.tq_codebook(d, b, seed=0, rotation=rot)
    enc = tq.tq_encode(q, dev(x, torch.bfloat16), chan=dev(chan, torch.int32), chan_rows=rows_per_group)
    rep = check_encode(*host(enc), xg, t)
    y = rng.standard_normal((3, d)).astype(np.float32)
    s = tq.tq_score(q, dev(y), 1, 3, enc, n).cpu().numpy()
    skip = rep.skip_rows.copy()
    check_scores(s, o.score(*o.prepare_query(y, t), rep.ref, t), rep.ref["norm"], np.linalg.norm(y, axis=1), d,
                 skip)
    assert np.all(s[:, 11] == 0.0)


# ------------------------------------------------------------------ on-the-fly S

@pytest.mark.parametrize("d,seed", [(128, 0), (64, 7), (96, 3), (1536, 0)])
def test_qjl_matrix_generated_on_device(tq, d, seed):
    """S generated on the device from the seed (TurboQuant article 2.3.2) is
    the oracle's S bit for bit: SplitMix64 stream 3, Box-Muller in double,
    one rounding to fp16."""
    q = tq.tq_codebook(d, 4, seed=seed)
    s = tq.tq_qjl_matrix(q).cpu().numpy().view(np.uint16)
    ref = o.qjl_matrix(d, d, seed).astype(np.float16).view(np.uint16)
    mism = int(np.count_nonzero(s != ref))
    assert mism == 0, f"{mism} of {s.size} entries differ"


@pytest.mark.parametrize("d", [128, 64])
def test_qjl_onthefly_bit_identical(tq, d):
    """With S generated inside the kernels (the bf16 Hadamard encode and the
    fused query preparation), codes, signs, norms and logits are bit-identical
    to the stored-S run, and the codes and logits still match the oracle."""
    rng = np.random.default_rng(d)
    n = 40000 + 77  # several tiles per CTA and a ragged last tile
    x = wl.to_bf16_values(rng.standard_normal((n, d)).astype(np.float32))
    x[5] = 0.0
    y = wl.to_bf16_values(rng.standard_normal((8, d)).astype(np.float32))
    q = tq.tq_codebook(d, 4, seed=0)
    xd = dev(x, torch.bfloat16)
    enc0 = tq.tq_encode(q, xd)
    s0 = tq.tq_score(q, dev(y), 2, 4, enc0, n // 2)
    tq.tq_set_qjl_onthefly(q, True)
    enc1 = tq.tq_encode(q, xd)
    s1 = tq.tq_score(q, dev(y), 2, 4, enc1, n // 2)
    tq.tq_set_qjl_onthefly(q, False)
    for a, b in ((enc0.codes, enc1.codes), (enc0.signs, enc1.signs), (enc0.norms, enc1.norms), (s0, s1)):
        assert torch.equal(a, b)
    t = tables(d, 4)
    rep = check_encode(*host(enc1), x, t)
    kpg = n // 2
    for g in range(2):
        rows = slice(g * kpg, (g + 1) * kpg)
        ref = {k: v[rows] for k, v in rep.ref.items()}
        yg = y[4 * g:4 * g + 4]
        check_scores(s1[4 * g:4 * g + 4].cpu().numpy(), o.score(*o.prepare_query(yg, t), ref, t), ref["norm"],
                     np.linalg.norm(yg, axis=1), d, rep.skip_rows[rows])


# ------------------------------------------------------------------ attention consumer

@pytest.mark.parametrize("d,b,G,nkeys,groups", [(128, 3, 4, 9000, 3), (64, 2, 3, 1001, 2), (128, 4, 8, 130, 5),
                                                 (128, 3, 16, 700, 1)])
def test_attend_against_oracle(tq, d, b, G, nkeys, groups):
    """Attention over a quantized cache: keys in inner-product mode scored
    by tq_score, values in TurboQuant-MSE mode.  The value codes are checked
    against the oracle's encode; tq_attend's output against the oracle's
    softmax over the same logits weighting the reconstructions of the same
    codes.  A key window that starts inside each group, ragged tiles, value
    norms over 2.6 decades.  Tolerance per coordinate: 2^-10 sum_k p_k ||v_k||
    (fp16 weights and centroids: two roundings of 2^-11 each) + 1e-6."""
    rng = np.random.default_rng(d * 10 + b + G)
    key_base = 17
    kpg = key_base + nkeys + 40
    n = groups * kpg
    kx = wl.to_bf16_values(rng.standard_normal((n, d)).astype(np.float32))
    vx = wl.to_bf16_values((rng.standard_normal((n, d)) * rng.uniform(0.05, 20.0, (n, 1))).astype(np.float32))
    y = wl.to_bf16_values(rng.standard_normal((groups * G, d)).astype(np.float32) * 2.0)
    qk = tq.tq_codebook(d, 4, seed=0)
    qv = tq.tq_codebook_mse(d, b, seed=0)
    kenc = tq.tq_encode(qk, dev(kx, torch.bfloat16))
    venc = tq.tq_encode(qv, dev(vx, torch.bfloat16))
    logits = tq.tq_score(qk, dev(y), groups, G, kenc, kpg)
    scale = 1.0 / math.sqrt(d)
    out = tq.tq_attend(qv, logits[:, key_base:], groups, G, venc, kpg, scale, key_base=key_base,
                       nkeys=nkeys).cpu().numpy()
    tv = tables_mse(d, b)
    codes, signs, norms = host(venc)
    check_encode(codes, signs, norms, vx, tv)
    from tests.layout import unpack_codes
    vcodes = unpack_codes(codes, d, tv.w)
    lg = logits.cpu().numpy().astype(np.float64)
    worst = 0.0
    for g in range(groups):
        rows = slice(g * kpg + key_base, g * kpg + key_base + nkeys)
        ve = {"codes": vcodes[rows], "norm": norms[rows, 0].astype(np.float64)}
        ls = lg[g * G:(g + 1) * G, key_base:key_base + nkeys]
        ref = o.attend(ls, scale, ve, tv)
        z = scale * ls
        p = np.exp(z - z.max(axis=1, keepdims=True))
        floor = (p / p.sum(axis=1, keepdims=True)) @ ve["norm"]
        err = np.abs(out[g * G:(g + 1) * G] - ref)
        bound = 2.0 ** -10 * floor[:, None] + 1e-6
        assert np.all(err <= bound), f"group {g}: worst {np.max(err / bound):.3f} of the bound"
        worst = max(worst, float(np.max(err / floor[:, None])))
    print(f"attend d={d} b={b} G={G}: worst error {worst:.2e} of sum p ||v||")


def test_attend_argument_checks(tq):
    """Unsupported value quantizers and bad windows are refused before any
    launch."""
    qv = tq.tq_codebook_mse(128, 3, seed=0)
    qk = tq.tq_codebook(128, 4, seed=0)  # inner-product mode: not a value quantizer here
    venc = tq.tq_encode(qv, torch.zeros((256, 128), dtype=torch.bfloat16, device="cuda"))
    logits = torch.zeros((4, 256), device="cuda")
    with pytest.raises(tq.TQError):
        tq.tq_attend(qk, logits, 1, 4, venc, 256, 0.1)
    with pytest.raises(tq.TQError):
        tq.tq_attend(qv, logits, 1, 4, venc, 256, 0.1, key_base=200, nkeys=100)
    with pytest.raises(tq.TQError):
        tq.tq_attend(qv, logits, 1, 4, venc, 256, float("nan"))
    out = tq.tq_attend(qv, logits, 1, 4, venc, 256, 0.1)  # zero values: zero output
    assert torch.all(out == 0)


@pytest.mark.parametrize("d,b,rot,G,mse", [(128, 4, "auto", 4, False), (96, 3, "auto", 4, False),
                                           (256, 3, "hadamard", 4, False), (128, 3, "auto", 60, False),
                                           (64, 2, "auto", 3, True)])
def test_score_in_two_halves(tq, d, b, rot, G, mse):
    """tq_score_prepare (on a side stream) then tq_score_prepared gives tq_score's
    logits bit for bit on every scoring route: the fused Hadamard query operand
    (d = 128), the separate operand (d = 96), the dense GEMM (d = 256), the CUDA
    cores (G = 60 > 48) and TurboQuant-MSE keys (m = 0).  One preparation serves
    two key sets; accumulate adds onto the output; the first case is also checked
    against the oracle."""
    groups, kpg = 3, 1000  # a ragged last tile
    rng = np.random.default_rng(d + G)
    x = rng.standard_normal((2, groups * kpg, d)).astype(np.float32)
    y = rng.standard_normal((groups * G, d)).astype(np.float32)
    q = tq.tq_codebook_mse(d, b, seed=0, rotation=rot) if mse else tq.tq_codebook(d, b, seed=0, rotation=rot)
    encs = [tq.tq_encode(q, dev(x[i])) for i in range(2)]
    yd = dev(y)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        ws = tq.tq_score_prepare(q, yd, groups, G, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    for enc in encs:
        ref = tq.tq_score(q, yd, groups, G, enc, kpg)
        got = tq.tq_score_prepared(q, groups, G, enc, kpg, ws)
        assert torch.equal(got, ref)
        tq.tq_score_prepared(q, groups, G, enc, kpg, ws, out=got, accumulate=True)
        assert torch.equal(got, ref + ref)
    if d == 128 and not mse:
        t = tables(d, b, rot)
        rep = check_encode(*host(encs[0]), x[0], t)
        s = tq.tq_score_prepared(q, groups, G, encs[0], kpg, ws).cpu().numpy()
        yt = o.prepare_query(y, t)
        for g in range(groups):
            rows, keys = slice(g * G, (g + 1) * G), slice(g * kpg, (g + 1) * kpg)
            r = {k: v[keys] for k, v in rep.ref.items()}
            check_scores(s[rows], o.score(yt[0][rows], yt[1][rows], r, t), r["norm"],
                         np.linalg.norm(y[rows], axis=1), d, rep.skip_rows[keys])


def test_back_to_back_steps(tq):
    """Steps of the split-precision KV layer (two gathered encodes, then two
    scorers, the second accumulating) queued back to back with no host
    synchronisation in between: no kernel records a failed wait, and the last
    step's logits equal those of the same calls run one at a time.  Then the
    scorer right after the encode that wrote its keys (tq_score_prepared on
    the same stream, no synchronisation) against the synchronised result."""
    n, groups, G = 32768, 8, 4
    xs = np.stack([wl.kv_head_keys(h, n) for h in range(groups)])
    x_dev = dev(xs.reshape(-1, 128), torch.bfloat16)
    y_dev = dev(wl.kv_queries())
    sel, rest = tq.tq_outlier_channels(x_dev, groups, n, 32)
    (da, ba), (db, bb) = wl.MIXED_SPLIT
    qa, qb = tq.tq_codebook(da, ba, seed=0), tq.tq_codebook(db, bb, seed=0)
    encs = [(qa.empty_encoded(groups * n), qb.empty_encoded(groups * n)) for _ in range(2)]
    out = torch.empty((groups * G, n), device="cuda")

    def step(i):
        (ea, eb), (ra, rb) = encs[i % 2], encs[(i + 1) % 2]
        tq.tq_encode(qa, x_dev, out=ea, chan=sel, chan_rows=n)
        tq.tq_encode(qb, x_dev, out=eb, chan=rest, chan_rows=n)
        tq.tq_score(qa, y_dev, groups, G, ra, n, out=out, ychan=sel)
        tq.tq_score(qb, y_dev, groups, G, rb, n, out=out, accumulate=True, ychan=rest)

    for i in range(6):
        step(i)
    tq.tq_sync_check(qa)
    tq.tq_sync_check(qb)
    got = out.clone()
    ra, rb = encs[(5 + 1) % 2]
    ref = tq.tq_score(qa, y_dev, groups, G, ra, n, ychan=sel)
    torch.cuda.synchronize()
    tq.tq_score(qb, y_dev, groups, G, rb, n, out=ref, accumulate=True, ychan=rest)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)

    q = tq.tq_codebook(128, 4, seed=0)
    ws = tq.tq_score_prepare(q, y_dev, groups, G)
    enc = q.empty_encoded(groups * n)
    enc.codes.zero_()
    tq.tq_encode(q, x_dev, out=enc)
    got = tq.tq_score_prepared(q, groups, G, enc, n, ws)
    tq.tq_sync_check(q)
    torch.cuda.synchronize()
    assert torch.equal(got, tq.tq_score(q, y_dev, groups, G, enc, n))

"""tq_score_noalloc: scores without a caller-provided workspace.

Some callers cannot give the library device memory for its scratch (the
device memory may belong to a framework's caching allocator, or an
allocation's synchronization may be unacceptable on their path).  For them
the library scores out of a fixed device buffer of its own.  This file checks
that entry point, called through the C ABI, on two calls in a row:

  - against the fp64 oracle's scores of the same keys and queries, within the
    score tolerance the parity tests use;
  - against tq_score (the entry point that takes a workspace): bit for bit
    where both run the same kernels (the integer tensor-core scorer, d <= 128),
    within the score tolerance where tq_score takes the tensor-core GEMM and
    this entry point the CUDA-core scorer (d > 128);
  - with accumulate = 1 and with a per-group query channel map (ychan).

The file is named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl
from oracle import tq_oracle as o
from tests.parity import check_encode, check_scores

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from online_vector_quantization_tq_b200 import build
    build.build()
    import online_vector_quantization_tq_b200 as pkg
    pkg.lib()
    return pkg


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(tq, q, y, groups, G, enc, kpg, out, accumulate=0, ychan=None):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return tq.lib().tq_score_noalloc(q.handle, _ptr(y), groups, G, y.stride(0), _ptr(ychan), _ptr(enc.codes),
                                     _ptr(enc.signs), _ptr(enc.norms), kpg, _ptr(out), accumulate, stream)


def _inputs(d, groups, G, kpg, seed, bf16):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((groups * kpg, d)).astype(np.float32)
    if bf16:
        x = wl.to_bf16_values(x)
    y = rng.standard_normal((groups * G, d)).astype(np.float32)
    return x, y


def _oracle_scores(t, x, y, groups, G, kpg, codes, signs, norms):
    """Per-group oracle logits, the keys' norms, and the keys whose scores are
    not comparable (boundary-exempt code differences)."""
    rep = check_encode(codes, signs, norms, x, t)
    ytil, p = o.prepare_query(y, t)
    ref = np.empty((groups * G, kpg))
    for g in range(groups):
        keys = slice(g * kpg, (g + 1) * kpg)
        enc_g = {k: v[keys] for k, v in rep.ref.items()}
        ref[g * G:(g + 1) * G] = o.score(ytil[g * G:(g + 1) * G], p[g * G:(g + 1) * G], enc_g, t)
    return ref, rep.ref["norm"], rep.skip_rows


def _check_groups(got, ref, xnorm, ynorm, skip, d, groups, G, kpg):
    for g in range(groups):
        rows, keys = slice(g * G, (g + 1) * G), slice(g * kpg, (g + 1) * kpg)
        check_scores(got[rows], ref[rows], xnorm[keys], ynorm[rows], d, skip[keys])


@pytest.mark.parametrize("d,b,rot,groups,G,kpg,bf16", [
    (128, 4, "auto", 3, 4, 2000, True),    # the kv shape: integer tensor-core scorer
    (96, 3, "auto", 2, 4, 1500, True),     # Haar d = 96, integer scorer
    (64, 3, "auto", 1, 16, 777, False),    # fp32 keys, ragged last key tile
    (384, 3, "haar", 2, 5, 1100, False),   # d > 128: CUDA-core scorer here, tensor-core GEMM in tq_score
])
def test_noalloc_against_oracle_and_workspace_scores(tq, d, b, rot, groups, G, kpg, bf16):
    x, y = _inputs(d, groups, G, kpg, seed=d + b, bf16=bf16)
    t = o.Tables(d, b, seed=0, rotation=rot)
    q = tq.tq_codebook(d, b, seed=0, rotation=rot)
    xd = torch.from_numpy(x).cuda()
    enc = tq.tq_encode(q, xd.to(torch.bfloat16) if bf16 else xd)
    yd = torch.from_numpy(y).cuda()
    ws_scores = tq.tq_score(q, yd, groups, G, enc, kpg)
    torch.cuda.synchronize()
    ref, xnorm, skip = _oracle_scores(t, x, y, groups, G, kpg, enc.codes.cpu().numpy(), enc.signs.cpu().numpy(),
                                      enc.norms.cpu().numpy())
    ynorm = np.linalg.norm(y, axis=1)
    same_kernels = d <= 128
    for call in range(2):  # two calls in a row share (and reuse) the fixed buffer
        out = torch.full_like(ws_scores, float("nan"))
        assert _noalloc(tq, q, yd, groups, G, enc, kpg, out) == 0
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got)), f"call {call}: unwritten scores"
        _check_groups(got, ref, xnorm, ynorm, skip, d, groups, G, kpg)
        if same_kernels:
            assert torch.equal(out, ws_scores), f"call {call}: differs from tq_score"
        else:
            _check_groups(got, ws_scores.cpu().numpy().astype(np.float64), xnorm, ynorm, skip, d, groups, G, kpg)


@pytest.mark.parametrize("d", [128, 384])
def test_noalloc_accumulate_and_query_channel_map(tq, d):
    """accumulate = 1 adds to the existing logits; ychan gathers each group's
    query channels (as the 3.5-bit split does) from wider query rows."""
    groups, G, kpg, width = 2, 4, 900, d + 32
    rot = "auto" if d == 128 else "haar"
    rng = np.random.default_rng(5 * d)
    x = rng.standard_normal((groups * kpg, d)).astype(np.float32)
    yw = rng.standard_normal((groups * G, width)).astype(np.float32)
    chan = np.stack([np.sort(rng.permutation(width)[:d]) for _ in range(groups)]).astype(np.int32)
    t = o.Tables(d, 3, seed=0, rotation=rot)
    q = tq.tq_codebook(d, 3, seed=0, rotation=rot)
    enc = tq.tq_encode(q, torch.from_numpy(x).cuda())
    yd = torch.from_numpy(yw).cuda()
    chan_d = torch.from_numpy(chan).cuda()
    base = torch.from_numpy(rng.standard_normal((groups * G, kpg)).astype(np.float32)).cuda()
    ws_scores = tq.tq_score(q, yd, groups, G, enc, kpg, out=base.clone(), accumulate=True, ychan=chan_d)
    torch.cuda.synchronize()
    y = np.concatenate([yw[g * G:(g + 1) * G][:, chan[g]] for g in range(groups)])
    ref, xnorm, skip = _oracle_scores(t, x, y, groups, G, kpg, enc.codes.cpu().numpy(), enc.signs.cpu().numpy(),
                                      enc.norms.cpu().numpy())
    ref = ref + base.cpu().numpy().astype(np.float64)
    ynorm = np.linalg.norm(y, axis=1)
    for call in range(2):
        out = base.clone()
        assert _noalloc(tq, q, yd, groups, G, enc, kpg, out, accumulate=1, ychan=chan_d) == 0
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        _check_groups(got, ref, xnorm, ynorm, skip, d, groups, G, kpg)
        if d <= 128:
            assert torch.equal(out, ws_scores), f"call {call}: differs from tq_score"
        else:
            _check_groups(got, ws_scores.cpu().numpy().astype(np.float64), xnorm, ynorm, skip, d, groups, G, kpg)


def test_noalloc_rejects_requests_beyond_the_buffer(tq):
    q = tq.tq_codebook(128, 4, seed=0)
    enc = tq.tq_encode(q, torch.randn(256, 128, device="cuda").to(torch.bfloat16))
    y = torch.randn(8192, 128, device="cuda")  # 8192 one-query groups need ~55 MiB of scratch
    out = torch.empty(8192, 1, device="cuda")
    assert _noalloc(tq, q, y, 8192, 1, enc, 1, out) == 7
    assert tq.lib().tq_status_string(7)

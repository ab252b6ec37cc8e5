"""tq_score_noalloc: scores without a caller-provided workspace.

Some callers cannot give the library device memory for its scratch (the
device memory may belong to a framework's caching allocator, or an
allocation's synchronization may be unacceptable on their path).  For them
the library scores out of a fixed device buffer of its own.  This file checks
that entry point, called through the C ABI, against tq_score (the entry point
that takes a workspace) on two calls in a row, each within the score
tolerance the parity tests use.  The file is named so that pytest collects it
last."""
import ctypes

import numpy as np
import pytest
import torch

from tests.parity import check_scores

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


@pytest.mark.parametrize("d,b,groups,G,kpg", [(128, 4, 3, 4, 2000), (96, 3, 2, 4, 1500), (64, 3, 1, 16, 777)])
def test_noalloc_matches_workspace_scores(tq, d, b, groups, G, kpg):
    torch.manual_seed(d + b)
    q = tq.tq_codebook(d, b, seed=0)
    x = torch.randn(groups * kpg, d, device="cuda").to(torch.bfloat16)
    y = torch.randn(groups * G, d, device="cuda")
    enc = tq.tq_encode(q, x)
    ref = tq.tq_score(q, y, groups, G, enc, kpg)
    torch.cuda.synchronize()
    xn = enc.norms[:, 0].cpu().numpy().reshape(groups, kpg)
    yn = torch.linalg.norm(y, dim=1).cpu().numpy().reshape(groups, G)
    ref_np = ref.cpu().numpy().astype(np.float64)
    for call in range(2):  # two calls in a row share (and reuse) the fixed buffer
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(tq, q, y, groups, G, enc, kpg, out) == 0
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got)), f"call {call}: unwritten scores"
        for g in range(groups):
            rows = slice(g * G, (g + 1) * G)
            check_scores(got[rows], ref_np[rows], xn[g], yn[g], d)


def test_noalloc_rejects_requests_beyond_the_buffer(tq):
    q = tq.tq_codebook(128, 4, seed=0)
    enc = tq.tq_encode(q, torch.randn(256, 128, device="cuda").to(torch.bfloat16))
    y = torch.randn(8192, 128, device="cuda")  # 8192 one-query groups need ~55 MiB of scratch
    out = torch.empty(8192, 1, device="cuda")
    assert _noalloc(tq, q, y, 8192, 1, enc, 1, out) == 7
    assert tq.lib().tq_status_string(7)

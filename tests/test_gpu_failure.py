"""The failure path of the tensor-core kernels, exercised without a fault or
a hang: a kernel whose bounded wait can never be satisfied gives up after
about 2 s, records its code in the quantizer's device error word, and the
host reads TQ_ERR_TIMEOUT; the context stays usable afterwards."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import online_vector_quantization_tq_b200 as m
    m.lib()
    return m


def test_bounded_wait_reports_timeout_and_context_survives(tq):
    q = tq.tq_codebook(128, 3, seed=0)
    tq.tq_sync_check(q)  # nothing pending
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    tq.tq_selftest_timeout(q)
    b.record()
    with pytest.raises(tq.TQError) as e:
        tq.tq_sync_check(q)
    assert e.value.code == 8
    # the bound is wall time on the GPU's global timer (2 s), not a count of
    # suspended tries, so the wait lasts about that long
    waited = a.elapsed_time(b) / 1e3
    assert 1.5 <= waited <= 10.0, f"bounded wait lasted {waited:.2f} s"
    tq.tq_sync_check(q)  # the check cleared the word
    # the context still runs the real path: encode + score, then a clean check
    rng = np.random.default_rng(5)
    x = torch.from_numpy(rng.standard_normal((2048, 128)).astype(np.float32)).cuda().to(torch.bfloat16)
    y = torch.from_numpy(rng.standard_normal((4, 128)).astype(np.float32)).cuda()
    enc = tq.tq_encode(q, x)
    s = tq.tq_score(q, y, 1, 4, enc, 2048)
    tq.tq_sync_check(q)
    assert torch.isfinite(s).all()

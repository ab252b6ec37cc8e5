"""Input generators: determinism, shapes, bf16 rounding against torch."""
import numpy as np
import torch

import workloads as w


def test_bf16_rounding_matches_torch():
    a = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 37.0
    a[:4] = [0.0, -0.0, 1e-30, 3.0e38]
    assert np.array_equal(w.to_bf16_values(a), torch.from_numpy(a).bfloat16().float().numpy())


def test_chunks_regenerate_bit_exactly():
    rows = np.array([5, 70000, 65535, 65536, 999_999])
    full = np.concatenate([w.ann_chunk(c, 1_000_000, 64) for c in (0, 1, 15)])
    got = w.ann_rows(rows, 1_000_000, 64)
    lut = {0: 0, 1: 65536, 15: 2 * 65536}
    for i, r in enumerate(rows):
        c = r // w.ANN_CHUNK
        assert np.array_equal(got[i], full[lut[c] + r - c * w.ANN_CHUNK])
    assert np.allclose(np.linalg.norm(got, axis=1), 1.0, atol=1e-6)


def test_kv_shapes_and_outliers():
    x = w.kv_head_keys(3, n=4096)
    ch = w.kv_outlier_channels(3)
    assert x.shape == (4096, 128) and ch.size == 4
    rms = np.sqrt(np.mean(x.astype(np.float64) ** 2, axis=0))
    assert np.all(rms[ch] > 8.0) and np.all(np.delete(rms, ch) < 1.2)
    assert np.array_equal(x, w.kv_head_keys(3, n=4096))
    assert np.array_equal(w.to_bf16_values(x), x)

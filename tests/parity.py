"""Parity rules shared by the GPU tests (test helper).

Codes and sign bits must equal the oracle's except where the oracle's own
fp64 value lies within EPS = 1e-6 of a decision boundary (a code threshold,
or 0 for a sign), in units of the normalized vector, and such exemptions may
cover at most 1e-4 of all coordinates.  A vector with an exempt code
difference has a different residual, so its sign bits and scores are not
compared (it is counted instead).  Scores must agree within 1e-3 relative,
measured against max(|s|, ||x|| ||y|| / sqrt(d)) so that near-zero logits are
not judged at unbounded relative precision."""
import math

import numpy as np

from oracle import tq_oracle as o
from tests.layout import unpack_codes, unpack_signs

EPS = 1e-6
MAX_EXEMPT_FRAC = 1e-4
SCORE_RTOL = 1e-3


class EncodeReport:
    def __init__(self, ref, skip_rows, n_code_exempt, n_sign_exempt):
        self.ref = ref
        self.skip_rows = skip_rows
        self.n_code_exempt = n_code_exempt
        self.n_sign_exempt = n_sign_exempt


def check_encode(codes_u8, signs_u8, norms, x, t: "o.Tables", ref=None) -> EncodeReport:
    """Compare one batch of GPU-encoded rows with the oracle's encoding of x."""
    if ref is None:
        ref = o.encode(x, t)
    codes = unpack_codes(codes_u8, t.d, t.w)
    bits = unpack_signs(signs_u8, t.m)
    cm = codes != ref["codes"]
    if cm.any():
        dist = o.boundary_distance(ref["u"], t)
        bad = cm & (dist >= EPS)
        assert not bad.any(), (f"{bad.sum()} code mismatches away from a boundary; first at "
                               f"{np.argwhere(bad)[:3].tolist()} dist={dist[bad][:3]}")
        assert np.all(np.abs(codes[cm] - ref["codes"][cm]) == 1)
    skip = np.any(cm, axis=1)
    sm = bits != ref["bits"]
    sm[skip] = False
    if sm.any():
        bad = sm & (np.abs(ref["z"]) >= EPS)
        assert not bad.any(), (f"{bad.sum()} sign mismatches with |z| >= {EPS}; "
                               f"z={ref['z'][bad][:5]}")
    total = cm.size + sm.size
    assert cm.sum() + sm.sum() <= MAX_EXEMPT_FRAC * total
    assert np.allclose(norms[:, 0], ref["norm"], rtol=3e-6, atol=1e-30)
    g_ok = ~skip
    assert np.allclose(norms[g_ok, 1], ref["gamma"][g_ok], rtol=2e-5, atol=2e-6)
    return EncodeReport(ref, skip | np.any(sm, axis=1), int(cm.sum()), int(sm.sum()))


def score_errors(s_gpu, s_ref, xnorm, ynorm, d, skip_keys=None):
    """Relative score errors against max(|s|, ||x|| ||y|| / sqrt(d)); where
    that is 0 (a zero key or query, whose score is exactly 0), the GPU score
    must be exactly 0 too (error 0, else inf)."""
    floor = np.outer(ynorm, xnorm) / math.sqrt(d)
    diff = np.abs(s_gpu.astype(np.float64) - s_ref)
    den = np.maximum(np.abs(s_ref), floor)
    with np.errstate(divide="ignore", invalid="ignore"):
        err = np.where(den > 0, diff / np.where(den > 0, den, 1.0), np.where(diff == 0, 0.0, np.inf))
    if skip_keys is not None and np.any(skip_keys):
        err[:, skip_keys] = 0.0
    return err


def check_scores(s_gpu, s_ref, xnorm, ynorm, d, skip_keys=None):
    err = score_errors(s_gpu, s_ref, xnorm, ynorm, d, skip_keys)
    worst = float(err.max()) if err.size else 0.0
    assert worst <= SCORE_RTOL, f"max relative score error {worst:.3e}"
    return worst


def check_topk(vals_gpu, idx_gpu, s_ref, xnorm, ynorm, d, k, skip_keys=None):
    """Top-k sets agree except for keys whose oracle score is within the score
    tolerance of the k-th score; returned scores match the oracle's scores of
    the returned keys; order is by descending score, ties by ascending index.
    Keys in skip_keys (a boundary-exempt code difference, so their GPU score
    is not the oracle's) are neither required nor score-checked."""
    nq, n = s_ref.shape
    skip = np.zeros(n, dtype=bool) if skip_keys is None else np.asarray(skip_keys, dtype=bool)
    for q in range(nq):
        order = np.lexsort((np.arange(n), -s_ref[q]))
        kth = s_ref[q, order[k - 1]]
        tol = SCORE_RTOL * max(abs(kth), ynorm[q] * np.max(xnorm) / math.sqrt(d))
        got = idx_gpu[q]
        assert len(set(got.tolist())) == k and np.all((got >= 0) & (got < n))
        ok = ~skip[got]
        assert np.all(s_ref[q, got[ok]] >= kth - 2 * tol)
        must = order[(s_ref[q, order] > kth + 2 * tol) & ~skip[order]]
        assert set(must.tolist()) <= set(got.tolist())
        check_scores(vals_gpu[q:q + 1, ok], s_ref[q:q + 1, got[ok]], xnorm[got[ok]], ynorm[q:q + 1], d)
        v = vals_gpu[q]
        assert np.all(np.diff(v) <= 0)
        for j in range(k - 1):
            if v[j] == v[j + 1]:
                assert got[j] < got[j + 1]

"""Pins for the fp64 oracle: each check compares it with something other than
itself -- published known answers, closed forms, a textbook table, library
routines, brute force, or statistics the method guarantees.  The planted-
mistake tests at the end show that plausible oracle bugs trip these pins."""
import math
import os

import mpmath
import numpy as np
import pytest
from scipy import integrate, linalg, special, stats

from oracle import tq_oracle as o


# ---------------------------------------------------------------- helpers

def _read_golden(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _gaussian_lloyd_max(w, iters=20000):
    """Lloyd-Max for N(0,1) from the Gaussian's own closed forms (independent
    of the oracle's Beta machinery): E[X | a<X<b] = (phi(a)-phi(b))/(Phi(b)-Phi(a))."""
    L = 1 << w
    thr = stats.norm.ppf(np.arange(1, L) / L)
    for _ in range(iters):
        lo = np.concatenate(([-np.inf], thr))
        hi = np.concatenate((thr, [np.inf]))
        c = (stats.norm.pdf(lo) - stats.norm.pdf(hi)) / (stats.norm.cdf(hi) - stats.norm.cdf(lo))
        thr = 0.5 * (c[:-1] + c[1:])
    lo = np.concatenate(([-np.inf], thr))
    hi = np.concatenate((thr, [np.inf]))
    p = stats.norm.cdf(hi) - stats.norm.cdf(lo)
    return c, thr, 1.0 - np.sum(c * c * p)


def _fwht_butterfly(v):
    """Unnormalized fast Walsh-Hadamard transform by in-place butterflies."""
    v = np.array(v, dtype=np.float64)
    h = 1
    n = v.shape[-1]
    while h < n:
        v = v.reshape(v.shape[:-1] + (n // (2 * h), 2, h))
        a = v[..., 0, :].copy()
        b = v[..., 1, :].copy()
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
        v = v.reshape(v.shape[:-3] + (n,))
        h *= 2
    return v


def _random_unit(n, d, seed):
    g = np.random.default_rng(seed).standard_normal((n, d))
    return g / np.linalg.norm(g, axis=1, keepdims=True)


# ---------------------------------------------------------------- RNG

def test_splitmix64_known_answers(golden_dir):
    for state, idx, out in _read_golden(os.path.join(golden_dir, "splitmix64_known_answers.txt")):
        got = int(o.splitmix64(int(state), np.array([int(idx)]))[0])
        assert got == int(out, 16)


def test_uniform_and_gaussian_laws():
    u = o.uniforms(o.stream_words(7, 3, 200000))
    assert stats.kstest(u, "uniform").pvalue > 1e-4
    g = o.gaussians(7, 3, 200000)
    assert abs(g.mean()) < 5 / math.sqrt(g.size)
    assert abs(g.var() - 1.0) < 5 * math.sqrt(2.0 / g.size)
    assert stats.kstest(g, "norm").pvalue > 1e-4
    # streams and seeds are decorrelated
    h = o.gaussians(7, 4, 200000)
    assert abs(np.corrcoef(g, h)[0, 1]) < 5 / math.sqrt(g.size)
    h2 = o.gaussians(8, 3, 200000)
    assert abs(np.corrcoef(g, h2)[0, 1]) < 5 / math.sqrt(g.size)


def test_rademacher_balance():
    s = o.rademacher(3, 0, 1 << 16)
    assert set(np.unique(s)) == {-1.0, 1.0}
    assert abs(s.mean()) < 5 / math.sqrt(s.size)


# ---------------------------------------------------------------- rotation

@pytest.mark.parametrize("d", [1, 2, 8, 32, 128, 256])
def test_hadamard_matches_library_sylvester(d):
    assert np.array_equal(o.hadamard(d) * math.sqrt(d), linalg.hadamard(d).astype(np.float64))
    h = o.hadamard(d)
    assert np.allclose(h @ h, np.eye(d), atol=1e-14)


@pytest.mark.parametrize("d", [8, 32, 128, 512])
def test_hadamard_rotation_against_butterflies(d):
    """R x equals three rounds of (sign flip, butterfly FWHT, 1/sqrt(d))."""
    r = o.rotation_matrix(d, seed=11)
    x = np.random.default_rng(1).standard_normal((5, d))
    v = x.copy()
    for stream in (o.STREAM_D1, o.STREAM_D2, o.STREAM_D3):
        v = _fwht_butterfly(v * o.rademacher(11, stream, d)) / math.sqrt(d)
    assert np.allclose(x @ r.T, v, rtol=0, atol=1e-12)


@pytest.mark.parametrize("d,kind", [(32, "hadamard"), (128, "hadamard"), (96, "haar"), (48, "haar")])
def test_rotation_preserves_norms(d, kind):
    r = o.rotation_matrix(d, seed=5, kind=kind)
    x = np.random.default_rng(2).standard_normal((64, d))
    nx = np.linalg.norm(x, axis=1)
    nr = np.linalg.norm(x @ r.T, axis=1)
    # exact in double for the Hadamard form; the Haar matrix is stored at fp32
    tol = 1e-14 if kind == "hadamard" else 3e-7
    assert np.max(np.abs(nr / nx - 1.0)) < tol
    assert np.max(np.abs(r.T @ r - np.eye(d))) < (1e-14 if kind == "hadamard" else 1e-6)


def test_haar_second_moment_over_seeds():
    """For a Haar matrix, E[R_ij^2] = 1/d and E[R_ij] = 0 (Haar invariance)."""
    d = 16
    vals = np.array([o.haar_matrix(d, s)[0, :] for s in range(600)])
    assert abs(np.mean(vals ** 2) - 1.0 / d) < 4 * np.std(vals ** 2) / math.sqrt(vals.size)
    assert abs(np.mean(vals)) < 4 * np.std(vals) / math.sqrt(vals.size)
    # without the sign fix the diagonal of R from QR would be biased positive;
    # here the first row's first entry has mean 0
    assert abs(np.mean(vals[:, 0])) < 4 * np.std(vals[:, 0]) / math.sqrt(vals.shape[0])


@pytest.mark.parametrize("d,kind", [(64, "hadamard"), (48, "haar")])
def test_rotated_coordinates_follow_beta_law(d, kind):
    """TurboQuant article 1.2.1 / 2.2.1: rotated coordinates of a unit vector
    follow Beta((d-1)/2, (d-1)/2) on [-1, 1].  Uses one fixed rotation on
    random unit vectors, so the law holds exactly for Haar and approximately
    (3 randomized Hadamard rounds) for the structured rotation."""
    r = o.rotation_matrix(d, seed=3, kind=kind)
    u = (_random_unit(4000, d, 9) @ r.T)[:, 0]
    assert stats.kstest(u, lambda x: o.coord_cdf(d, x)).pvalue > 1e-3


# ---------------------------------------------------------------- codebook

@pytest.mark.parametrize("d", [3, 8, 32, 128, 1536])
def test_coordinate_density_is_normalized(d):
    s = 1.0 / math.sqrt(d)
    tot = integrate.quad(lambda x: o.coord_pdf(d, x), -1, 1, points=[-s, 0.0, s], limit=200)[0]
    assert abs(tot - 1.0) < 1e-10
    for x in (-0.5 * s, 0.3 * s, min(2.0 * s, 0.9)):
        cdf = integrate.quad(lambda t: o.coord_pdf(d, t), -1, x, points=[0.0] if x > 0 else None, limit=200)[0]
        assert abs(cdf - o.coord_cdf(d, x)) < 1e-10


@pytest.mark.parametrize("d", [3, 4, 8, 64, 128, 1536])
def test_one_bit_closed_form(d):
    c, t, mse = o.lloyd_max(d, 1)
    with mpmath.workdps(40):  # Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
        e_abs = float(mpmath.gamma(mpmath.mpf(d) / 2) / (mpmath.sqrt(mpmath.pi) * mpmath.gamma(mpmath.mpf(d + 1) / 2)))
    assert np.allclose(c, [-e_abs, e_abs], rtol=1e-13, atol=0)
    assert t.tolist() == [0.0]
    assert abs(mse - (1.0 / d - e_abs ** 2)) < 1e-15


@pytest.mark.parametrize("w", [1, 2, 3, 4])
def test_uniform_case_d3(w):
    """d = 3: the density is flat on [-1, 1], so Lloyd-Max is the uniform quantizer."""
    c, t, mse = o.lloyd_max(3, w)
    L = 1 << w
    assert np.allclose(c, -1.0 + (2 * np.arange(L) + 1) / L, atol=1e-13)
    assert np.allclose(t, -1.0 + 2.0 * np.arange(1, L) / L, atol=1e-13)
    assert abs(mse - 1.0 / (3 * 4 ** w)) < 1e-14


@pytest.mark.parametrize("d,w", [(8, 2), (32, 4), (96, 2), (128, 2), (128, 3), (1536, 3)])
def test_lloyd_max_fixed_point_by_quadrature(d, w):
    """Centroids are conditional means of their bins (by adaptive quadrature of
    the density, independent of the oracle's closed forms) and thresholds are
    midpoints; the printed MSE equals the quadrature distortion."""
    c, t, mse = o.lloyd_max(d, w)
    edges = np.concatenate(([-1.0], t, [1.0]))
    scale = 1.0 / math.sqrt(d)
    dist = 0.0
    for i in range(c.size):
        lo, hi = edges[i], edges[i + 1]
        pts = [p for p in (-8 * scale, -scale, 0.0, scale, 8 * scale) if lo < p < hi]
        mass = integrate.quad(lambda x: o.coord_pdf(d, x), lo, hi, points=pts or None, limit=400, epsabs=0, epsrel=1e-13)[0]
        mom = integrate.quad(lambda x: x * o.coord_pdf(d, x), lo, hi, points=pts or None, limit=400, epsabs=0, epsrel=1e-13)[0]
        assert abs(mom / mass - c[i]) < 1e-11 * scale
        dist += integrate.quad(lambda x: (x - c[i]) ** 2 * o.coord_pdf(d, x), lo, hi, points=pts or None, limit=400, epsabs=0, epsrel=1e-12)[0]
    assert np.allclose(t, 0.5 * (c[:-1] + c[1:]), rtol=0, atol=1e-16)
    assert abs(dist - mse) < 1e-10 * mse
    assert np.all(np.diff(c) > 0) and np.allclose(c, -c[::-1], atol=1e-16)


def test_gaussian_limit_textbook_table(golden_dir):
    """The Gaussian Lloyd-Max quantizer computed from the Gaussian's closed forms
    matches Max (1960), and sqrt(d)-scaled codebooks approach it as d grows."""
    rows = _read_golden(os.path.join(golden_dir, "gaussian_lloyd_max_max1960.txt"))
    table = {}
    for bits, kind, *vals in rows:
        table[(int(bits), kind)] = np.array([float(v) for v in vals])
    for w in (1, 2, 3, 4):
        gc, gt, gm = _gaussian_lloyd_max(w)
        L = 1 << w
        assert np.allclose(gc[L // 2:], table[(w, "out")], rtol=2e-3, atol=0)
        assert abs(gm - table[(w, "mse")][0]) < 2e-3 * gm
        if (w, "thr") in table:
            assert np.allclose(gt[L // 2:], table[(w, "thr")], rtol=2e-3, atol=0)
        errs = []
        for d in (256, 4096, 65536):
            c, t, mse = o.lloyd_max(d, w)
            errs.append(np.max(np.abs(c * math.sqrt(d) - gc)))
            assert abs(mse * d - gm) < 40.0 / d
        assert errs[2] < errs[1] < errs[0] and errs[2] < 1e-3


@pytest.mark.parametrize("d", [8, 32, 96, 128, 1536])
@pytest.mark.parametrize("w", [1, 2, 3, 4])
def test_distortion_bound(d, w):
    """TurboQuant article 3.1: MSE within 2.7 times the Shannon bound 4^-R per
    unit vector (R = w bits per coordinate), i.e. d * D_w <= 2.7 * 4^-w."""
    _, _, mse = o.lloyd_max(d, w)
    assert d * mse <= 2.7 * 4.0 ** (-w)
    assert d * mse >= 4.0 ** (-w)  # no quantizer beats the Shannon bound


# ---------------------------------------------------------------- encode

def test_rotation_direction():
    """u = R x_hat: a vector x = R^T v (v unit) must rotate back to v."""
    t = o.Tables(32, 3, seed=4)
    v = _random_unit(3, 32, 5)
    x = 2.5 * v @ t.R  # rows: (R^T v)^T = v^T R
    enc = o.encode(x, t)
    assert np.allclose(enc["u"], v, atol=1e-13)
    assert np.allclose(enc["norm"], 2.5, rtol=1e-14)


@pytest.mark.parametrize("w", [1, 2, 3])
def test_brute_force_codes_d8(w):
    """d = 8: the chosen codes minimise ||u - c[codes]|| over all (2^w)^8 code
    vectors, and gamma is that minimum."""
    d = 8
    t = o.Tables(d, w + 1, seed=6)
    L = 1 << w
    grid = np.stack(np.meshgrid(*([np.arange(L)] * d), indexing="ij"), axis=-1).reshape(-1, d)
    pts = t.centroids[grid]
    x = np.random.default_rng(w).standard_normal((3 if w == 3 else 6, d))
    enc = o.encode(x, t)
    for i in range(x.shape[0]):
        dist = np.sum((pts - enc["u"][i]) ** 2, axis=1)
        best = np.argmin(dist)
        assert np.array_equal(grid[best], enc["codes"][i])
        assert abs(math.sqrt(dist[best]) - enc["gamma"][i]) < 1e-14
    # per coordinate, the code is the nearest centroid (brute force over the
    # codebook, no thresholds involved), on many vectors
    xs = np.random.default_rng(100 + w).standard_normal((20000, d))
    enc = o.encode(xs, t)
    near = np.argmin(np.abs(enc["u"][..., None] - t.centroids), axis=-1)
    assert np.array_equal(near, enc["codes"])


@pytest.mark.parametrize("d,b,kind", [(64, 3, "hadamard"), (128, 4, "hadamard"), (48, 3, "haar")])
def test_encode_mse_matches_lloyd_max(d, b, kind):
    """E ||x_hat - R^T c[codes]||^2 over random unit vectors = d * D_w (4 sigma)."""
    t = o.Tables(d, b, seed=8, rotation=kind)
    x = _random_unit(20000, d, 12)
    enc = o.encode(x, t)
    rec = t.centroids[enc["codes"]] @ t.R  # R^T c
    err = np.sum((x - rec) ** 2, axis=1)
    assert np.allclose(err, enc["gamma"] ** 2, rtol=1e-6, atol=1e-12)
    assert abs(err.mean() - d * t.coord_mse) < 4 * err.std() / math.sqrt(err.size)


def test_zero_vector_and_threshold_tie():
    t = o.Tables(32, 3, seed=1)
    enc = o.encode(np.zeros((1, 32)), t)
    L = 1 << t.w
    assert enc["norm"][0] == 0.0
    assert np.all(enc["codes"] == L // 2 - 1)  # u == 0 == middle threshold -> lower code
    y = np.random.default_rng(0).standard_normal((2, 32))
    s = o.score(*o.prepare_query(y, t), enc, t)
    assert np.all(s == 0.0)
    # a coordinate exactly on a threshold takes the lower code
    u = np.full((1, 32), t.thresholds[-1])
    assert np.all(np.searchsorted(t.thresholds, u, side="left") == L - 2)


def test_sign_bits_and_gamma_definition():
    t = o.Tables(16, 3, seed=2)
    x = np.random.default_rng(3).standard_normal((50, 16))
    enc = o.encode(x, t)
    r = enc["u"] - t.centroids[enc["codes"]]
    z = r @ t.S.T
    assert np.array_equal(enc["bits"], z >= 0)
    assert np.allclose(enc["gamma"], np.linalg.norm(r, axis=1), rtol=1e-15)


def test_qjl_matrix_is_fp16_gaussian():
    s = o.qjl_matrix(128, 128, 0)
    assert np.array_equal(s, s.astype(np.float16).astype(np.float64))
    g = o.gaussians(0, o.STREAM_S, 128 * 128).reshape(128, 128)
    assert np.max(np.abs(s - g)) <= np.max(np.abs(g)) * 2.0 ** -11


# ---------------------------------------------------------------- estimator

def _estimates_over_S(d, b, nseeds, x, y, rot_seed=1):
    t = o.Tables(d, b, seed=rot_seed)
    ests, var = [], None
    for s in range(nseeds):
        t.S = o.qjl_matrix(t.m, d, 1000 + s)
        enc = o.encode(x, t)
        ytil, p = o.prepare_query(y, t)
        ests.append(o.score(ytil, p, enc, t)[0, 0])
        if var is None:
            var = o.estimator_variance(ytil, enc, t)[0, 0]
    return np.array(ests), var


def test_estimator_unbiased_over_S():
    """TurboQuant article 1.2.3: the two-stage estimate is unbiased.  With R
    fixed, the mean over independent draws of S equals <y, x> within 4 sigma,
    and the spread matches the closed-form variance."""
    d, b, N = 32, 3, 6000
    rng = np.random.default_rng(21)
    x = rng.standard_normal((1, d))
    y = rng.standard_normal((1, d))
    ests, var = _estimates_over_S(d, b, N, x, y)
    truth = float(x[0] @ y[0])
    assert abs(ests.mean() - truth) < 4 * math.sqrt(var / N)
    # variance of the variance estimate: 2 var^2 / N for near-Gaussian samples
    assert abs(ests.var() - var) < 6 * var * math.sqrt(2.0 / N)


def test_estimator_decomposition():
    """<y~, c[codes]> + <y~, r> = <R y, R x_hat> = <y, x_hat>: the MSE term plus
    the exact residual term recovers the true inner product (R orthogonal)."""
    d = 32
    t = o.Tables(d, 3, seed=9)
    x = np.random.default_rng(1).standard_normal((4, d))
    enc = o.encode(x, t)
    y = np.random.default_rng(2).standard_normal((3, d))
    ytil, p = o.prepare_query(y, t)
    mse_term = ytil @ t.centroids[enc["codes"]].T
    r = enc["u"] - t.centroids[enc["codes"]]
    xhat = x / np.linalg.norm(x, axis=1, keepdims=True)
    assert np.allclose(mse_term + ytil @ r.T, y @ xhat.T, atol=1e-12)
    # and the estimate's QJL term uses p = S R y
    assert np.allclose(p, y @ t.R.T @ t.S.T, atol=1e-10)


# ---------------------------------------------------------------- top-k, outliers

def test_topk_against_selection():
    rng = np.random.default_rng(5)
    s = np.round(rng.standard_normal((4, 300)), 1)  # many exact ties
    val, idx = o.topk(s, 10)
    for q in range(4):
        left = list(range(300))
        for j in range(10):
            best = max(left, key=lambda i: (s[q, i], -i))
            assert idx[q, j] == best and val[q, j] == s[q, best]
            left.remove(best)


def test_outlier_channels():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((5000, 128))
    planted = [3, 40, 77, 120]
    x[:, planted] *= 10.0
    sel = o.outlier_channels(x, 32)
    assert set(planted) <= set(sel.tolist()) and sel.size == 32
    ms = np.mean(x * x, axis=0)
    assert np.min(ms[sel]) >= np.max(np.delete(ms, sel))
    tie = np.ones((10, 8))
    assert o.outlier_channels(tie, 3).tolist() == [0, 1, 2]


# ---------------------------------------------------------------- planted mistakes

def test_planted_mistakes_are_caught(monkeypatch):
    """Plausible oracle bugs each fail one of the pins above."""
    # 1. transposed rotation
    real_rot = o.rotation_matrix
    monkeypatch.setattr(o, "rotation_matrix", lambda d, seed, kind="auto": real_rot(d, seed, kind).T)
    with pytest.raises(AssertionError):
        test_hadamard_rotation_against_butterflies(32)
    monkeypatch.setattr(o, "rotation_matrix", real_rot)

    # 1b. encode applying R^T instead of R
    real_encode = o.encode

    def transposed_encode(x, t):
        class T2:
            pass
        t2 = T2()
        t2.__dict__.update(t.__dict__)
        t2.R = t.R.T
        return real_encode(x, t2)
    monkeypatch.setattr(o, "encode", transposed_encode)
    with pytest.raises(AssertionError):
        test_rotation_direction()
    monkeypatch.setattr(o, "encode", real_encode)

    # 2. missing sqrt(pi/2) in the estimator (QJL term biased)
    real_score = o.score

    def bad_score(ytil, p, enc, t):
        sig = np.where(enc["bits"], 1.0, -1.0)
        return enc["norm"][None, :] * (ytil @ t.centroids[enc["codes"]].T
                                       + (p @ sig.T) * enc["gamma"][None, :] / t.m)
    monkeypatch.setattr(o, "score", bad_score)
    with pytest.raises(AssertionError):
        test_estimator_unbiased_over_S()
    monkeypatch.setattr(o, "score", real_score)

    # 3. inverted sign bits

    def flipped(x, t):
        e = real_encode(x, t)
        e["bits"] = ~e["bits"]
        return e
    monkeypatch.setattr(o, "encode", flipped)
    with pytest.raises(AssertionError):
        test_estimator_unbiased_over_S()
    with pytest.raises(AssertionError):
        test_sign_bits_and_gamma_definition()
    monkeypatch.setattr(o, "encode", real_encode)

    # 4. codebook: thresholds at the wrong place (off-by-one centroid pairing)
    real_lm = o.lloyd_max

    def bad_lm(d, w, **kw):
        c, t, m = real_lm(d, w, **kw)
        return c, 0.5 * (c[:-1] + c[1:]) * 1.01, m
    monkeypatch.setattr(o, "lloyd_max", bad_lm)
    with pytest.raises(AssertionError):
        test_lloyd_max_fixed_point_by_quadrature(32, 4)
    with pytest.raises(AssertionError):
        test_brute_force_codes_d8(2)
    monkeypatch.setattr(o, "lloyd_max", real_lm)

    # 5. a dropped sign diagonal in the structured rotation
    real_rad = o.rademacher
    monkeypatch.setattr(o, "rademacher", lambda s, st, d: np.ones(d) if st == 1 else real_rad(s, st, d))
    r_bad = o.rotation_matrix(32, 11)
    monkeypatch.setattr(o, "rademacher", real_rad)
    x = np.random.default_rng(1).standard_normal((5, 32))
    v = x.copy()
    for stream in (o.STREAM_D1, o.STREAM_D2, o.STREAM_D3):
        v = _fwht_butterfly(v * o.rademacher(11, stream, 32)) / math.sqrt(32)
    assert not np.allclose(x @ r_bad.T, v, atol=1e-12)


# ---------------------------------------------------------------- boundary distance

def _brute_boundary_distance(u, thresholds):
    """min over every threshold t_i of |u - t_i|, by enumeration."""
    u = np.asarray(u, dtype=np.float64)
    return np.min(np.abs(u[..., None] - np.asarray(thresholds)[None, :]), axis=-1)


@pytest.mark.parametrize("d,b", [(128, 2), (128, 4), (96, 3), (32, 5), (8, 3)])
def test_boundary_distance_brute_force(d, b):
    """The exemption rule's distance (what the GPU parity tests forgive) is the
    distance to the nearest Lloyd-Max threshold (article 1.2.2: a code changes
    only where u crosses a threshold).  Checked against enumeration on random
    u, on u exactly at every threshold, just below / above each, below t_0 and
    above t_last (including |u| = 1)."""
    t = o.Tables(d, b, seed=3)
    thr = t.thresholds
    rng = np.random.default_rng(d * 10 + b)
    u = rng.uniform(-1.0, 1.0, size=(200, 7)) * rng.choice([1.0, 0.1, 0.01], size=(200, 1))
    assert np.array_equal(o.boundary_distance(u, t), _brute_boundary_distance(u, thr))
    eps = 1e-9
    special_u = np.concatenate([thr, thr - eps, thr + eps, [thr[0] - 0.5, thr[-1] + 0.5, -1.0, 1.0, 0.0]])
    got = o.boundary_distance(special_u, t)
    assert np.array_equal(got, _brute_boundary_distance(special_u, thr))
    assert np.all(got[:thr.size] == 0.0)
    assert np.allclose(got[thr.size:3 * thr.size], eps, rtol=1e-6) or thr.size == 1
    # for these u the distance is to the NEAREST threshold: the outer tails
    # measure to t_0 / t_last, not to a neighbour
    assert got[3 * thr.size] == pytest.approx(0.5)
    assert got[3 * thr.size + 1] == pytest.approx(0.5)
    assert got[3 * thr.size + 2] == pytest.approx(1.0 + thr[0])
    assert got[3 * thr.size + 3] == pytest.approx(1.0 - thr[-1])


def test_boundary_distance_planted_off_by_one(monkeypatch):
    """An off-by-one in the neighbour index (measuring to t_{j+1} instead of
    t_j) widens or misplaces the exemption window; the brute-force pin fails."""
    real = o.boundary_distance

    def off_by_one(u, t):
        j = np.searchsorted(t.thresholds, u)
        lo = np.abs(u - t.thresholds[np.clip(j, 0, t.thresholds.size - 1)])
        hi = np.abs(u - t.thresholds[np.clip(j + 1, 0, t.thresholds.size - 1)])
        return np.minimum(lo, hi)
    monkeypatch.setattr(o, "boundary_distance", off_by_one)
    with pytest.raises(AssertionError):
        test_boundary_distance_brute_force(128, 4)
    monkeypatch.setattr(o, "boundary_distance", real)


# ---------------------------------------------------------------- TurboQuant-MSE mode

@pytest.mark.parametrize("b", [1, 2, 3])
def test_mse_mode_brute_force_d8(b):
    """MSE mode gives all b bits to the codebook: at d = 8 the codes minimise
    ||u - c[codes]|| over all (2^b)^8 code vectors; no sign bits; the score is
    ||x|| <y~, c[codes]> (the brute-force nearest codebook point)."""
    d = 8
    t = o.Tables(d, b, seed=4, mode="mse")
    assert t.w == b and t.m == 0 and t.S.shape == (0, d)
    L = 1 << b
    grid = np.stack(np.meshgrid(*([np.arange(L)] * d), indexing="ij"), axis=-1).reshape(-1, d)
    pts = t.centroids[grid]
    x = np.random.default_rng(b).standard_normal((4, d))
    y = np.random.default_rng(50 + b).standard_normal((3, d))
    enc = o.encode(x, t)
    assert enc["bits"].shape == (4, 0)
    for i in range(x.shape[0]):
        best = np.argmin(np.sum((pts - enc["u"][i]) ** 2, axis=1))
        assert np.array_equal(grid[best], enc["codes"][i])
    ytil, p = o.prepare_query(y, t)
    assert p.shape == (3, 0)
    s = o.score(ytil, p, enc, t)
    want = (y @ t.R.T) @ (t.centroids[enc["codes"]] * np.linalg.norm(x, axis=1)[:, None]).T
    assert np.allclose(s, want, rtol=1e-13, atol=1e-13)


def test_mse_mode_shrinks_inner_products_by_one_minus_d_D():
    """Over random Haar rotations the TurboQuant-MSE estimate averages to
    (1 - d D_b) <y, x> (centroids are bin means); at b = 1 and large d the
    factor tends to 2/pi.  Checked by simulation for fixed x, y at d = 24."""
    d, b, trials = 24, 2, 3000
    t = o.Tables(d, b, seed=0, mode="mse", rotation="haar")
    rng = np.random.default_rng(9)
    x = rng.standard_normal(d)
    y = 0.6 * x + rng.standard_normal(d)  # correlated with x, so <y, x> is far from 0
    est = np.empty(trials)
    for s in range(trials):
        t.R = o.rotation_matrix(d, 1000 + s, "haar")
        enc = o.encode(x[None, :], t)
        est[s] = o.score(*o.prepare_query(y[None, :], t), enc, t)[0, 0]
    want = o.mse_inner_product_gain(t) * float(y @ x)
    assert abs(est.mean() - want) < 4.0 * est.std() / math.sqrt(trials)
    # and the factor differs from 1 by far more than that error: the bias is real
    assert abs(float(y @ x) - want) > 8.0 * est.std() / math.sqrt(trials)
    # b = 1, large d: 1 - d D_1 -> 2/pi (d D_1 -> 1 - 2/pi for the sign quantizer)
    _, _, mse = o.lloyd_max(4096, 1)
    assert abs((1.0 - 4096 * mse) - 2.0 / math.pi) < 2e-4


def test_mse_mode_distortion_and_planted_shrinkage_mistake(monkeypatch):
    """MSE mode encodes with distortion d D_b per unit vector (like the
    inner-product mode's codebook stage), and a gain formula missing its d
    factor fails the shrinkage pin."""
    d, b = 64, 3
    t = o.Tables(d, b, seed=2, mode="mse")
    x = _random_unit(20000, d, 3)
    enc = o.encode(x, t)
    err = np.sum((x - t.centroids[enc["codes"]] @ t.R) ** 2, axis=1)
    se = err.std() / math.sqrt(err.size)
    assert abs(err.mean() - d * t.coord_mse) < 4 * se
    monkeypatch.setattr(o, "mse_inner_product_gain", lambda tt: 1.0 - tt.coord_mse)
    with pytest.raises(AssertionError):
        test_mse_mode_shrinks_inner_products_by_one_minus_d_D()


# ---------------------------------------------------------------- two-stage retrieval

def test_rerank_equals_exact_topk_when_candidates_cover_it():
    """With every key a candidate, the second stage is the exact top-k of the
    raw inner products (brute force by full sort); with a candidate subset
    it is the exact top-k of that subset; duplicate candidates and empty
    slots (-1) do not change the result; equal scores go to the lower key."""
    rng = np.random.default_rng(31)
    x = rng.standard_normal((300, 24))
    x[200] = x[17]  # an exact tie between keys 17 and 200
    y = rng.standard_normal((5, 24))
    y[0] = x[17]
    every = np.tile(np.arange(300), (5, 1))
    val, idx = o.rerank(y, x, every, 7)
    exact = y @ x.T
    for q in range(5):
        order = sorted(range(300), key=lambda i: (-exact[q, i], i))[:7]
        assert idx[q].tolist() == order
        assert np.allclose(val[q], exact[q, order], rtol=1e-15, atol=0)
    assert idx[0][:2].tolist() == [17, 200]
    sub = rng.choice(300, size=(5, 40), replace=True)
    sub[:, :3] = -1
    val2, idx2 = o.rerank(y, x, sub, 5)
    for q in range(5):
        cs = sorted(set(sub[q][sub[q] >= 0].tolist()), key=lambda i: (-exact[q, i], i))[:5]
        assert idx2[q].tolist() == cs


def test_rerank_planted_mistake(monkeypatch):
    """A stage that keeps the k smallest instead of the k largest fails."""
    real = o.rerank
    monkeypatch.setattr(o, "rerank", lambda y, x, c, k: real(-y, x, c, k))
    with pytest.raises(AssertionError):
        test_rerank_equals_exact_topk_when_candidates_cover_it()


# ---------------------------------------------------------------- attention consumer

def test_dequantize_distortion_norms_and_zero_rows():
    """The reconstruction ||x|| R^T c[codes] has squared error d D_b per unit
    of ||x||^2 on random vectors of any norm (the Lloyd-Max distortion of the
    codebook stage), and a zero row reconstructs to zero.  A reconstruction
    with R in place of R^T, or without the norm, fails."""
    d, b = 64, 3
    t = o.Tables(d, b, seed=4, mode="mse")
    x = _random_unit(20000, d, 5) * np.exp(np.random.default_rng(6).uniform(-3, 3, (20000, 1)))
    x[7] = 0.0
    enc = o.encode(x, t)
    xh = o.dequantize(enc, t)
    assert np.all(xh[7] == 0.0)
    keep = np.arange(x.shape[0]) != 7
    rel = np.sum((x - xh) ** 2, axis=1)[keep] / np.sum(x * x, axis=1)[keep]
    assert abs(rel.mean() - d * t.coord_mse) < 4 * rel.std() / math.sqrt(rel.size)
    wrong_r = enc["norm"][:, None] * (t.centroids[enc["codes"]] @ t.R.T)
    assert np.mean(np.sum((x - wrong_r) ** 2, axis=1)[keep] / np.sum(x * x, axis=1)[keep]) > 0.5
    no_norm = t.centroids[enc["codes"]] @ t.R
    assert np.mean(np.sum((x - no_norm) ** 2, axis=1)[keep] / np.sum(x * x, axis=1)[keep]) > 0.5


def test_attend_special_cases():
    """Softmax attention over dequantized values: a single key returns its
    reconstruction whatever the logit; equal logits return the mean of the
    reconstructions; adding a constant to a query's logits changes nothing;
    a logit far above the others returns that key's reconstruction; the
    scale multiplies the logits."""
    d, b = 32, 3
    t = o.Tables(d, b, seed=8, mode="mse")
    rng = np.random.default_rng(9)
    v = rng.standard_normal((50, d)) * rng.uniform(0.1, 10.0, (50, 1))
    enc = o.encode(v, t)
    vh = o.dequantize(enc, t)
    one = {k: a[:1] for k, a in enc.items()}
    assert np.allclose(o.attend(rng.standard_normal((3, 1)) * 50, 0.7, one, t), vh[:1], rtol=1e-13, atol=0)
    assert np.allclose(o.attend(np.full((2, 50), 3.25), 1.0, enc, t), np.mean(vh, axis=0)[None, :].repeat(2, 0),
                       rtol=1e-12, atol=1e-14)
    s = rng.standard_normal((4, 50)) * 3
    base = o.attend(s, 0.5, enc, t)
    assert np.allclose(o.attend(s + np.array([[1.0], [-7.0], [30.0], [0.5]]), 0.5, enc, t), base, rtol=1e-12,
                       atol=1e-13)
    assert np.allclose(o.attend(2.0 * s, 0.25, enc, t), base, rtol=1e-12, atol=1e-13)
    dom = s.copy()
    dom[1, 17] = 2000.0
    assert np.allclose(o.attend(dom, 1.0, enc, t)[1], vh[17], rtol=1e-12, atol=1e-13)


def test_attend_planted_mistakes(monkeypatch):
    """A softmax taken over the queries instead of the keys, or one that
    ignores the scale, fails the special cases."""
    real = o.attend

    def over_queries(logits, scale, v_enc, t_v):
        z = scale * np.asarray(logits, dtype=np.float64)
        w = np.exp(z - z.max(axis=0, keepdims=True))
        return (w / w.sum(axis=0, keepdims=True)) @ o.dequantize(v_enc, t_v)

    monkeypatch.setattr(o, "attend", over_queries)
    with pytest.raises(AssertionError):
        test_attend_special_cases()
    monkeypatch.setattr(o, "attend", lambda lg, sc, e, t: real(lg, 1.0, e, t))
    with pytest.raises(AssertionError):
        test_attend_special_cases()

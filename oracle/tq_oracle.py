"""Plain fp64 CPU oracle for TurboQuant-style online vector quantization.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only the tests, the smoke check in ``__graft_entry__`` and
the CPU-baseline leg of ``bench.py`` use it.  It shares no code with the CUDA
library (``online_vector_quantization_tq_b200``); the two meet only through the
seeded input generators of the ``workloads`` package, which hold none of the
method's arithmetic.

Sources.  "TurboQuant article" below is the intelliparadigm.com page
"TurboQuant 技术概览与核心价值" (sections 1.2.1-1.2.3, 2.1-2.3, 3.1, 4.2.2);
"TurboQuant blog" is the blog.hotdry.top page "TurboQuant 深度解读" (sections
三 and 四).  Each function names the section it restates.  Where the pages are
silent or garbled, the reading taken is stated in the docstring.

Every step follows the method's plain definition in float64, with library
primitives (matmul, QR, sort, the regularized incomplete beta function) as
single steps; there is no blocking, fusion or reordering beyond that.

Parity status per function (the pins live in ``tests/test_oracle_pins.py``):
  splitmix64 / gaussians / rademacher ... pinned (published known answers,
                                          moments, KS test)
  hadamard / rotation_matrix ............ pinned (library Hadamard, H H = I,
                                          norm preservation, Haar moments)
  lloyd_max ............................. pinned (closed forms at w=1 and d=3,
                                          Gaussian large-d limit, textbook
                                          Gaussian table, fixed-point residual,
                                          2.7 * 4^-w distortion bound)
  encode ................................ pinned (brute force at d=8, MSE vs
                                          Lloyd-Max distortion, exact
                                          re-encoding of codebook points)
  prepare_query / score ................. pinned (unbiasedness over seeds of S,
                                          closed-form variance)
  topk .................................. pinned (against an independent
                                          brute-force selection)
  rerank (two-stage retrieval) .......... pinned (exact top-k by full sort
                                          when every key is a candidate,
                                          subsets, ties, planted mistake)
  TurboQuant-MSE mode (mode="mse") ...... pinned (brute force at d=8, MSE
                                          against D_b, the shrinkage factor
                                          1 - d D_b over random rotations,
                                          and its 2/pi limit at b = 1)
  dequantize ............................ pinned (codebook points are
                                          reconstructed exactly, distortion
                                          d D_b over random vectors)
  attend (attention consumer) ........... pinned (one key, equal logits =
                                          mean, shift invariance, a dominant
                                          logit, planted mistakes)
  outlier_channels ...................... pinned (planted outliers, ties)
  boundary_distance ..................... pinned (enumeration over every
                                          threshold, exact-threshold and
                                          tail cases, planted off-by-one)
  End-to-end scores on the pages' own workloads: parity unpinned -- the pages
  print no worked numeric example.
"""
from __future__ import annotations

import functools
import math

import mpmath
import numpy as np
from scipy import special

# ---------------------------------------------------------------------------
# Random draws.  The pages draw with numpy's RandomState (TurboQuant article,
# 2.1.2 and 2.3.2); that generator is not a contract, so both this oracle and
# the CUDA library implement one published counter-based generator instead:
# SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
# generators", OOPSLA 2014), indexed directly by counter.
# ---------------------------------------------------------------------------

_M64 = (1 << 64) - 1
GOLDEN_GAMMA = 0x9E3779B97F4A7C15

# Streams of the quantizer's random draws.
STREAM_D1, STREAM_D2, STREAM_D3, STREAM_S, STREAM_HAAR = 0, 1, 2, 3, 4


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function (variant 13 of Stafford's mixers)."""
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def splitmix64(state: int, index: np.ndarray) -> np.ndarray:
    """Output ``index`` (0-based) of SplitMix64 started from ``state``.

    The generator adds the golden gamma to its state before each output and
    returns the mixed state, so output k is mix64(state + (k+1)*gamma).
    """
    index = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(state & _M64) + (index + np.uint64(1)) * np.uint64(GOLDEN_GAMMA)
    return _mix64(z)


def stream_words(seed: int, stream: int, count: int) -> np.ndarray:
    """``count`` 64-bit words of stream ``stream`` for quantizer seed ``seed``.

    The stream key is output ``stream`` of SplitMix64 started from ``seed``;
    the stream's words are the outputs of SplitMix64 started from that key.
    """
    key = int(splitmix64(seed, np.array([stream]))[0])
    return splitmix64(key, np.arange(count, dtype=np.uint64))


def uniforms(words: np.ndarray) -> np.ndarray:
    """53-bit uniforms in [0, 1) from the top bits of each word."""
    return (words >> np.uint64(11)).astype(np.float64) * 2.0 ** -53


def gaussians(seed: int, stream: int, count: int) -> np.ndarray:
    """``count`` N(0,1) draws by the Box-Muller transform (cosine branch).

    Draw i uses words 2i and 2i+1: u1 = (top53(w_2i) + 1) * 2^-53 in (0, 1],
    u2 = top53(w_2i+1) * 2^-53, g = sqrt(-2 ln u1) * cos(2 pi u2).
    """
    w = stream_words(seed, stream, 2 * count)
    u1 = ((w[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53
    u2 = uniforms(w[1::2])
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def rademacher(seed: int, stream: int, d: int) -> np.ndarray:
    """Random +-1 diagonal: entry j is -1 when bit 0 of word j is set."""
    w = stream_words(seed, stream, d)
    return np.where((w & np.uint64(1)) != 0, -1.0, 1.0)


# ---------------------------------------------------------------------------
# Rotation (TurboQuant article 1.2.1 and 2.1.1-2.1.2)
# ---------------------------------------------------------------------------

def hadamard(d: int) -> np.ndarray:
    """Orthonormal Sylvester Walsh-Hadamard matrix: H_ij = (-1)^popcount(i&j)/sqrt(d).

    TurboQuant article 2.1.2 applies an unspecified ``fwht``; the reading taken
    is the orthonormal transform in natural (Sylvester) order.
    """
    if d < 1 or d & (d - 1):
        raise ValueError("Hadamard rotation needs a power-of-two dimension")
    i = np.arange(d)
    parity = np.zeros((d, d), dtype=np.int64)
    a = i[:, None] & i[None, :]
    while np.any(a):
        parity ^= a & 1
        a = a >> 1
    return np.where(parity == 1, -1.0, 1.0) / math.sqrt(d)


def haar_matrix(d: int, seed: int) -> np.ndarray:
    """Seeded Haar-distributed orthogonal matrix, rounded to fp32 and promoted.

    TurboQuant article 1.2.1: QR of a d x d standard Gaussian matrix.  The page
    omits the sign correction; without it Q is not Haar distributed, so Q is
    multiplied by sign(diag(R)).  The stored matrix is fp32 (both sides use the
    same fp32 values), promoted back to float64 here.
    """
    g = gaussians(seed, STREAM_HAAR, d * d).reshape(d, d)
    q, r = np.linalg.qr(g)
    q = q * np.where(np.diag(r) < 0, -1.0, 1.0)[None, :]
    return q.astype(np.float32).astype(np.float64)


def rotation_matrix(d: int, seed: int, kind: str = "auto") -> np.ndarray:
    """The quantizer's rotation R as an explicit d x d float64 matrix.

    Power-of-two d ("hadamard"): three rounds of (+-1 diagonal, then
    orthonormal Walsh-Hadamard), R = H D3 H D2 H D1 (TurboQuant article 2.1.2;
    its 2.1.1 formula is garbled, the three-round form is taken).  The signs
    are drawn once per seed, not per call.  Other d ("haar"): ``haar_matrix``.
    """
    if kind == "auto":
        kind = "hadamard" if d & (d - 1) == 0 else "haar"
    if kind == "hadamard":
        h = hadamard(d)
        r = np.eye(d)
        for stream in (STREAM_D1, STREAM_D2, STREAM_D3):
            r = h @ (rademacher(seed, stream, d)[:, None] * r)
        return r
    if kind == "haar":
        return haar_matrix(d, seed)
    raise ValueError(f"unknown rotation kind {kind!r}")


def qjl_matrix(m: int, d: int, seed: int) -> np.ndarray:
    """QJL projection S (m x d): seeded N(0,1) entries stored at fp16 precision.

    TurboQuant article 2.3.2 draws ``randn(k, len(r))``; the projection is
    fixed per seed (drawn once, m = d rows).  Entries are the Box-Muller
    Gaussians of stream S, row-major, rounded once to the nearest fp16 value.
    """
    g = gaussians(seed, STREAM_S, m * d).reshape(m, d)
    return g.astype(np.float16).astype(np.float64)


# ---------------------------------------------------------------------------
# Scalar codebook (TurboQuant article 1.2.2, 2.2.1-2.2.2, 3.1)
# ---------------------------------------------------------------------------

def _beta_a(d: int) -> float:
    # Coordinates of a uniform unit vector: X = 2T - 1 with T ~ Beta(a, a),
    # a = (d-1)/2, i.e. density proportional to (1 - x^2)^((d-3)/2) on [-1, 1].
    return (d - 1) / 2.0


@functools.lru_cache(maxsize=None)
def _log_normalizer(a: float) -> float:
    """log B(1/2, a), the log of the integral of (1 - x^2)^(a-1) over [-1, 1],
    in 30-digit arithmetic (double-precision log-gamma differences lose about
    1e-12 relative accuracy at a ~ 800)."""
    with mpmath.workdps(30):
        return float(mpmath.log(mpmath.beta(mpmath.mpf(1) / 2, mpmath.mpf(a))))


def coord_cdf(d: int, x: np.ndarray) -> np.ndarray:
    a = _beta_a(d)
    x = np.clip(np.asarray(x, dtype=np.float64), -1.0, 1.0)
    return special.betainc(a, a, (1.0 + x) / 2.0)


def coord_sf(d: int, x: np.ndarray) -> np.ndarray:
    """P(X > x), computed without cancellation in the upper tail."""
    a = _beta_a(d)
    x = np.clip(np.asarray(x, dtype=np.float64), -1.0, 1.0)
    return special.betainc(a, a, (1.0 - x) / 2.0)


def coord_pdf(d: int, x: np.ndarray) -> np.ndarray:
    a = _beta_a(d)
    x = np.asarray(x, dtype=np.float64)
    logz = _log_normalizer(a)
    xc = np.clip(x, -1.0, 1.0)
    with np.errstate(divide="ignore"):
        return np.where(np.abs(x) < 1.0,
                        np.exp((a - 1.0) * np.log1p(-xc * xc) - logz), 0.0)


def _bin_mass(d: int, lo: np.ndarray, hi: np.ndarray) -> np.ndarray:
    # Upper-tail form on the positive side, lower-tail form on the negative
    # side, so tail bins keep full relative precision.
    pos = lo >= 0.0
    m_pos = coord_sf(d, lo) - coord_sf(d, hi)
    m_neg = coord_cdf(d, hi) - coord_cdf(d, lo)
    return np.where(pos, m_pos, m_neg)


def _bin_first_moment(d: int, lo: np.ndarray, hi: np.ndarray) -> np.ndarray:
    # Integral of x f(x) over [lo, hi] in closed form:
    # d/dx [-(1-x^2)^a / (2a Z)] = x (1-x^2)^(a-1) / Z.
    a = _beta_a(d)
    logz = _log_normalizer(a)

    def g(x):
        with np.errstate(divide="ignore"):
            return np.where(np.abs(x) < 1.0,
                            np.exp(a * np.log1p(-x * x) - logz), 0.0) / (2.0 * a)
    return g(lo) - g(hi)


def lloyd_max(d: int, w: int, tol: float = 1e-14, max_iter: int = 100000):
    """(centroids, thresholds, per-coordinate MSE) of the w-bit Lloyd-Max quantizer.

    TurboQuant article 1.2.2 iterates centroids <-> boundaries on the rotated
    coordinate's density, and 2.2.1 identifies that density as
    Beta((d-1)/2, (d-1)/2); it is used exactly here rather than fitted from
    samples (2.2.2).  Readings: equal-probability initial bins; thresholds are
    midpoints of adjacent centroids; centroids are the conditional means of
    their bins; the codebook is kept symmetric; stop when no centroid moves by
    more than ``tol`` times the largest centroid.
    MSE = E[X^2] - sum_i c_i^2 P(bin i), with E[X^2] = 1/d.
    """
    if d < 3 or w < 1:
        raise ValueError("need d >= 3 and w >= 1")
    levels = 1 << w
    q = np.arange(1, levels) / levels
    a = _beta_a(d)
    thr = 2.0 * special.betaincinv(a, a, q) - 1.0
    cen = np.zeros(levels)
    for _ in range(max_iter):
        lo = np.concatenate(([-1.0], thr))
        hi = np.concatenate((thr, [1.0]))
        new = _bin_first_moment(d, lo, hi) / _bin_mass(d, lo, hi)
        new = 0.5 * (new - new[::-1])
        done = np.max(np.abs(new - cen)) <= tol * np.max(np.abs(new))
        cen = new
        thr = 0.5 * (cen[:-1] + cen[1:])
        if done:
            break
    lo = np.concatenate(([-1.0], thr))
    hi = np.concatenate((thr, [1.0]))
    mse = 1.0 / d - float(np.sum(cen * cen * _bin_mass(d, lo, hi)))
    return cen, thr, mse


# ---------------------------------------------------------------------------
# Quantizer tables
# ---------------------------------------------------------------------------

class Tables:
    """Everything a (d, b, m, seed, rotation, mode) quantizer fixes, in float64.

    mode "prod" (the default): b - 1 bits to the Lloyd-Max codebook and one
    QJL bit per coordinate (the inner-product quantizer, TurboQuant article
    1.2.3).  mode "mse": TurboQuant-MSE, all b bits to the Lloyd-Max codebook
    and no QJL stage (article 4.1.1 recommends it for most heads at 3 bits,
    4.2.1 quantizes a vector index with it); there is no S and m = 0."""

    def __init__(self, d: int, b: int, m: int | None = None, seed: int = 0,
                 rotation: str = "auto", mode: str = "prod"):
        if mode not in ("prod", "mse"):
            raise ValueError(f"unknown mode {mode!r}")
        self.mode = mode
        self.d, self.b = d, b
        self.w = b if mode == "mse" else b - 1
        self.m = 0 if mode == "mse" else (d if m is None else m)
        self.seed = seed
        self.R = rotation_matrix(d, seed, rotation)
        self.S = qjl_matrix(self.m, d, seed) if mode == "prod" else np.zeros((0, d))
        self.centroids, self.thresholds, self.coord_mse = lloyd_max(d, self.w)


# ---------------------------------------------------------------------------
# Encode (TurboQuant article 1.2.3, 2.3.1-2.3.2, 4.2.1)
# ---------------------------------------------------------------------------

def encode(x: np.ndarray, t: Tables) -> dict:
    """Encode rows of ``x`` (n x d, any float dtype, promoted exactly to fp64).

    1. norm = ||x||, x_hat = x / norm (x_hat = 0 for a zero vector);  the norm
       is stored beside the codes (TurboQuant article 4.2.1).
    2. u = R x_hat (article 1.2.1).
    3. code_j = #{i : t_i < u_j} for the (b-1)-bit Lloyd-Max thresholds
       (article 1.2.2-1.2.3); a value equal to a threshold takes the lower code.
    4. r = u - c[code] in the rotated domain (article 2.3.1), gamma = ||r||.
    5. z = S r, sign bit = [z >= 0] (article 2.3.2; np.sign's 0 is read as +1).
    Returns the intermediate u and z too, for boundary-exemption accounting.
    """
    x = np.asarray(x, dtype=np.float64)
    norm = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(norm > 0.0, norm, 1.0)
    xhat = np.where(norm[:, None] > 0.0, x / safe[:, None], 0.0)
    u = xhat @ t.R.T
    codes = np.searchsorted(t.thresholds, u, side="left")
    r = u - t.centroids[codes]
    gamma = np.sqrt(np.sum(r * r, axis=1))
    z = r @ t.S.T  # (n, 0) in TurboQuant-MSE mode: no sign bits
    bits = z >= 0.0
    return {"codes": codes.astype(np.int64), "bits": bits, "norm": norm,
            "gamma": gamma, "u": u, "z": z}


# ---------------------------------------------------------------------------
# Query side and estimator (TurboQuant article 1.2.3, 4.2.2; blog 三)
# ---------------------------------------------------------------------------

def prepare_query(y: np.ndarray, t: Tables):
    """Rotated query y~ = R y (article 4.2.2: apply the same rotation) and its
    QJL projection p = S y~, both in fp64."""
    y = np.asarray(y, dtype=np.float64)
    ytil = y @ t.R.T
    p = ytil @ t.S.T
    return ytil, p


def score(ytil: np.ndarray, p: np.ndarray, enc: dict, t: Tables) -> np.ndarray:
    """Asymmetric inner-product estimate for every (query, key) pair.

    s = ||x|| * ( <y~, c[codes]> + gamma * sqrt(pi/2)/m * <p, 2*bit - 1> ).
    The first term is the MSE stage; the second is the QJL estimate of
    <y~, r>, unbiased because E[(s.q) sign(s.r)] = sqrt(2/pi) <q, r>/||r||
    for a Gaussian row s (article 1.2.3 states the unbiasedness; the pages
    print no constant, so it is derived here).  Returns an nq x n array.
    """
    chat = t.centroids[enc["codes"]]
    mse_term = ytil @ chat.T
    if t.m == 0:
        # TurboQuant-MSE (article 4.1.1, 4.2.1): the codebook term alone;
        # biased, E_R[s] = (1 - d D_b) <y, x> (see mse_inner_product_gain)
        return enc["norm"][None, :] * mse_term
    sig = np.where(enc["bits"], 1.0, -1.0)
    qjl_term = (p @ sig.T) * (enc["gamma"][None, :] * math.sqrt(math.pi / 2.0) / t.m)
    return enc["norm"][None, :] * (mse_term + qjl_term)


def mse_inner_product_gain(t: Tables) -> float:
    """E over the rotation of the TurboQuant-MSE estimate divided by <y, x>.

    For a Lloyd-Max codebook every centroid is the mean of its bin, so
    E[u c(u)] = E[c(u)^2] = E[u^2] - D = 1/d - D per coordinate.  By the
    rotation's symmetry E_R[R^T c(R x)] is a multiple a x of x, and
    a = E<u, c(u)> = 1 - d D for a unit x: the estimate shrinks every inner
    product by the factor 1 - d D_b (the bias the article contrasts with the
    unbiased inner-product quantizer, 1.2.3)."""
    return 1.0 - t.d * t.coord_mse


def estimator_variance(ytil: np.ndarray, enc: dict, t: Tables) -> np.ndarray:
    """Closed-form variance of the estimate over the draw of S, given R.

    Var = ||x||^2 gamma^2 / m * ((pi/2) ||y~||^2 - <y~, r/gamma>^2), from
    E[(s.q)^2] = ||q||^2 and the mean above, for m independent rows.
    """
    r = enc["u"] - t.centroids[enc["codes"]]
    g = enc["gamma"]
    rn = r / np.where(g > 0, g, 1.0)[:, None]
    yy = np.sum(ytil * ytil, axis=1)
    yr = ytil @ rn.T
    return (enc["norm"] ** 2 * g ** 2)[None, :] / t.m * (math.pi / 2.0 * yy[:, None] - yr ** 2)


def topk(scores: np.ndarray, k: int):
    """Top-k per row of ``scores``: descending score, ties to the lower index
    (article 4.2.2 first stage).  A full stable sort, then the first k."""
    nq, n = scores.shape
    k = min(k, n)
    idx = np.empty((nq, k), dtype=np.int64)
    val = np.empty((nq, k), dtype=np.float64)
    for q in range(nq):
        order = np.lexsort((np.arange(n), -scores[q]))
        idx[q] = order[:k]
        val[q] = scores[q, order[:k]]
    return val, idx


# ---------------------------------------------------------------------------
# Mixed-precision KV split (TurboQuant article 3.2 and 4.1.1; blog 四)
# ---------------------------------------------------------------------------

def outlier_channels(x_head: np.ndarray, count: int) -> np.ndarray:
    """Indices of the ``count`` highest-RMS channels of one head's keys.

    The article keeps about 25% of channels as outliers at higher precision
    (4.1.1; 3.5 bits in 3.2).  Reading: RMS over all keys of the head in fp64,
    ties to the lower channel index; returned in ascending channel order.
    """
    x = np.asarray(x_head, dtype=np.float64)
    ms = np.mean(x * x, axis=0)
    order = np.lexsort((np.arange(ms.size), -ms))
    return np.sort(order[:count])


def boundary_distance(u: np.ndarray, t: Tables) -> np.ndarray:
    """Distance of each rotated coordinate to its nearest decision threshold."""
    j = np.searchsorted(t.thresholds, u)
    lo = np.abs(u - t.thresholds[np.clip(j - 1, 0, t.thresholds.size - 1)])
    hi = np.abs(u - t.thresholds[np.clip(j, 0, t.thresholds.size - 1)])
    return np.minimum(lo, hi)


# ---------------------------------------------------------------------------
# Two-stage retrieval (TurboQuant article 4.2.2)
# ---------------------------------------------------------------------------

def dequantize(enc: dict, t: Tables) -> np.ndarray:
    """Reconstruction from the codebook stage: x_hat = ||x|| R^T c[codes].

    The codes select centroids of the rotated, normalised coordinates
    (article 1.2.2); rotating back and restoring the stored norm (article
    4.2.1) gives the TurboQuant-MSE estimate of x (article 4.1.2 dequantizes
    the cache this way before attention).  Row form: c[codes] @ R."""
    c = t.centroids[enc["codes"]]
    return enc["norm"][:, None] * (c @ t.R)


def attend(logits: np.ndarray, scale: float, v_enc: dict, t_v: Tables) -> np.ndarray:
    """Attention output of queries over a quantized KV cache: the softmax
    over keys of scale * logits, weighting the dequantized values.

    Article 4.1.1 quantizes both keys and values of the cache (the size
    formula counts both) and recommends TurboQuant-MSE for most heads;
    article 4.1.2 dequantizes before the attention product.  The pages give
    no further definition of the value path.  Reading: values are encoded
    by the same quantizer family in TurboQuant-MSE mode, and the output is
    softmax(scale * logits) @ dequantize(values), in fp64; the logits are
    the keys' inner-product estimates (``score``).  ``logits`` is nq x n,
    the result nq x d."""
    z = scale * np.asarray(logits, dtype=np.float64)
    z = z - z.max(axis=1, keepdims=True)
    w = np.exp(z)
    w = w / w.sum(axis=1, keepdims=True)
    return w @ dequantize(v_enc, t_v)


def rerank(y: np.ndarray, x: np.ndarray, cand: np.ndarray, k: int):
    """Second stage of two-stage retrieval: the candidates a first stage on
    the quantized vectors returned are re-scored exactly and the k best kept.

    Article 4.2.2 describes quickly screening a top-K on the quantized
    vectors, then refining that candidate set; the refinement's measure is
    not printed.  Reading: the exact inner product <y, x> with the stored
    raw vectors, in fp64 here; ties to the lower key index; candidate
    indices < 0 are empty slots.  ``x`` holds the raw database rows indexed
    by ``cand`` (nq x kc).  Returns (scores, indices), each nq x k, padded
    with (-inf, -1) when a row has fewer than k valid candidates."""
    y = np.asarray(y, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    nq = y.shape[0]
    val = np.full((nq, k), -np.inf)
    idx = np.full((nq, k), -1, dtype=np.int64)
    for q in range(nq):
        c = np.unique(cand[q][cand[q] >= 0])  # ascending: ties go to the lower index
        s = x[c] @ y[q]
        order = np.lexsort((c, -s))[:k]
        val[q, :order.size] = s[order]
        idx[q, :order.size] = c[order]
    return val, idx

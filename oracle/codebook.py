"""Lloyd-Max codebook for one rotated coordinate (oracle, float64).

After a uniformly random rotation, each coordinate of a unit vector in R^d
follows

    f(x) = Gamma(d/2) / (sqrt(pi) * Gamma((d-1)/2)) * (1 - x^2)^((d-3)/2),  x in [-1, 1]

[tq.net, "TurboQuant 两阶段算法 / PolarQuant：极坐标变换", 坐标分布公式]; the page
[ttakun, "为什么随机旋转是整个算法的底层杠杆"] names this law (Beta-shaped, tending to a
Gaussian in high d) and says the optimal scalar quantizer for it is precomputed
once with the Lloyd-Max algorithm ([tq.net, "实现步骤草图", 预计算 Lloyd-Max 质心]).

Two independent routes compute the codebook:

* ``lloyd_max``: closed forms.  X = 2B - 1 with B ~ Beta(a, a), a = (d-1)/2, so
  the CDF is the regularized incomplete beta I_{(1+t)/2}(a, a); the first
  moment of a bin has the antiderivative -(1-x^2)^((d-1)/2) / (d-1) times the
  normalising constant.
* ``lloyd_max_quadrature``: the same fixed-point iteration with both bin
  integrals done by Gauss-Legendre quadrature of f and x*f.

Reading (the pages are silent on the stopping rule): iterate to the float64
fixed point.  Tie rule used everywhere: a value exactly on a threshold takes
the upper cell.

Parity: pinned by the d = 3 closed form (uniform law -> uniform quantizer, MSE
4^-b), the b = 1 closed form (centroid E|X|), the Gaussian large-d limit
(J. Max, 1960), agreement of the two routes, and symmetry.
"""
from __future__ import annotations

import math

import mpmath
import numpy as np
from scipy import special, stats


def _log_norm_const(d: int) -> float:
    """log of Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)), evaluated at 40 digits: in
    float64 the difference of two lgamma values near 4e3 (d = 1536) would carry
    a relative error of ~5e-13 into every first moment."""
    with mpmath.workdps(40):
        v = mpmath.loggamma(mpmath.mpf(d) / 2) - mpmath.log(mpmath.pi) / 2 \
            - mpmath.loggamma(mpmath.mpf(d - 1) / 2)
        return float(v)


def coord_pdf(x, d: int):
    """The coordinate density f(x) above (d >= 3)."""
    x = np.asarray(x, dtype=np.float64)
    return np.exp(_log_norm_const(d)) * np.power(np.clip(1.0 - x * x, 0.0, None), (d - 3) / 2.0)


def coord_cdf(t, d: int):
    """P[X <= t] = I_{(1+t)/2}(a, a), a = (d-1)/2.  Upper tail by symmetry for accuracy."""
    t = np.asarray(t, dtype=np.float64)
    a = (d - 1) / 2.0
    lo = special.betainc(a, a, np.clip((1.0 + t) / 2.0, 0.0, 1.0))
    hi = 1.0 - special.betainc(a, a, np.clip((1.0 - t) / 2.0, 0.0, 1.0))
    return np.where(t <= 0.0, lo, hi)


def _bin_mass(lo, hi, d: int):
    """P[lo < X <= hi], computed from the nearer tail to keep relative accuracy."""
    a = (d - 1) / 2.0
    lo = np.asarray(lo, dtype=np.float64)
    hi = np.asarray(hi, dtype=np.float64)
    left = special.betainc(a, a, (1.0 + hi) / 2.0) - special.betainc(a, a, (1.0 + lo) / 2.0)
    right = special.betainc(a, a, (1.0 - lo) / 2.0) - special.betainc(a, a, (1.0 - hi) / 2.0)
    return np.where(hi <= 0.0, left, np.where(lo >= 0.0, right, left))


def bin_first_moment(lo, hi, d: int):
    """Integral of x f(x) over [lo, hi] = C/(d-1) * ((1-lo^2)^((d-1)/2) - (1-hi^2)^((d-1)/2))."""
    lo = np.asarray(lo, dtype=np.float64)
    hi = np.asarray(hi, dtype=np.float64)
    c = math.exp(_log_norm_const(d)) / (d - 1)
    p = (d - 1) / 2.0
    # (1-a^2)^p - (1-b^2)^p evaluated as e^B * expm1(A - B) with A, B = p*log1p(-x^2):
    # the plain power loses ~p ulps of 1-x^2, which the difference of two
    # nearly equal terms would turn into a large relative error.
    with np.errstate(divide="ignore"):
        A = p * np.log1p(-np.minimum(lo * lo, 1.0))
        B = p * np.log1p(-np.minimum(hi * hi, 1.0))
    big = np.maximum(A, B)
    small = np.minimum(A, B)
    sgn = np.where(A >= B, 1.0, -1.0)
    diff = np.where(np.isneginf(big), 0.0,
                    np.exp(big) * -np.expm1(np.where(np.isneginf(small), -np.inf, small - big)))
    return c * sgn * diff


def _initial_centroids(b: int, d: int) -> np.ndarray:
    k = 2 ** b
    return stats.norm.ppf((np.arange(k) + 0.5) / k) / math.sqrt(d)


def _thresholds(c: np.ndarray) -> np.ndarray:
    return 0.5 * (c[:-1] + c[1:])


def _iterate(b: int, d: int, moments, max_iter: int) -> tuple[np.ndarray, np.ndarray]:
    c = _initial_centroids(b, d)
    best, since_best = np.inf, 0
    for _ in range(max_iter):
        t = _thresholds(c)
        edges = np.concatenate(([-1.0], t, [1.0]))
        m0, m1 = moments(edges[:-1], edges[1:])
        c_new = m1 / m0
        # symmetrise exactly (the law is even); keeps c_k = -c_{K-1-k} bit-exact
        c_new = 0.5 * (c_new - c_new[::-1])
        step = float(np.max(np.abs(c_new - c)))
        c = c_new
        # float64 fixed point: the step sits at the rounding floor of the bin
        # integrals and has not shrunk for 200 iterations
        if step < best:
            best, since_best = step, 0
        else:
            since_best += 1
        if step == 0.0 or since_best >= 200:
            break
    return c, _thresholds(c)


def lloyd_max(b: int, d: int, max_iter: int = 20000) -> tuple[np.ndarray, np.ndarray]:
    """Centroids c[2^b] (ascending) and thresholds t[2^b - 1] = midpoints, closed-form route."""
    if d < 3 or not (1 <= b <= 8):
        raise ValueError("need d >= 3 and 1 <= b <= 8")
    return _iterate(b, d, lambda lo, hi: (_bin_mass(lo, hi, d), bin_first_moment(lo, hi, d)), max_iter)


def lloyd_max_quadrature(b: int, d: int, nodes: int = 400, max_iter: int = 20000):
    """Same fixed point, bin integrals by Gauss-Legendre quadrature (independent route).

    Each bin is clipped to [lo, min(hi, lo + 14/sqrt(d))] on the outer bins: the
    mass beyond 14 standard deviations is below 1e-40 and does not change the
    float64 result."""
    xg, wg = np.polynomial.legendre.leggauss(nodes)
    width = 14.0 / math.sqrt(d)

    def moments(lo, hi):
        m0 = np.empty(len(lo))
        m1 = np.empty(len(lo))
        for i, (a, bb) in enumerate(zip(lo, hi)):
            a2 = max(a, bb - width) if a == -1.0 else a
            b2 = min(bb, a + width) if bb == 1.0 else bb
            if a == -1.0 and bb == 1.0:
                a2, b2 = -1.0, 1.0
            xs = 0.5 * (b2 - a2) * xg + 0.5 * (b2 + a2)
            ws = 0.5 * (b2 - a2) * wg
            fx = coord_pdf(xs, d)
            m0[i] = np.sum(ws * fx)
            m1[i] = np.sum(ws * xs * fx)
        return m0, m1

    return _iterate(b, d, moments, max_iter)


def distortion(c: np.ndarray, d: int) -> float:
    """D(b, d) = E||y - Q(y)||^2 for a uniform unit vector y: d * (1/d - sum_k c_k^2 P_k)
    (Lloyd centroid condition E[X Q(X)] = E[Q(X)^2])."""
    t = _thresholds(c)
    edges = np.concatenate(([-1.0], t, [1.0]))
    p = _bin_mass(edges[:-1], edges[1:], d)
    return float(1.0 - d * np.sum(c * c * p))


def b1_centroid(d: int) -> float:
    """Closed form of the 1-bit centroid: E|X| = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))."""
    return math.exp(math.lgamma(d / 2.0) - 0.5 * math.log(math.pi) - math.lgamma((d + 1) / 2.0))

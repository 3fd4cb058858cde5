"""PolarQuant, the polar stage-one variant of TurboQuant -- oracle, float64.

Pages: [tmdm, "双剑合璧：PolarQuant + QJL", ✦ PolarQuant]: after the random
rotation the Cartesian coordinates become a radius and a chain of angles;
angles are bounded, so no per-vector normalisation constants are stored, and
with QJL on top the cache lands near 3 bits per element.  [admirer, "第一階段"]:
the coordinates are grouped in pairs and mapped to polar form; the pair radii
are gathered and transformed the same way, recursively, until one final
radius and a set of angles remain; after the rotation the angles follow
concentrated (Beta-type) laws and each part is quantized with its own
high-quality scalar quantizer on a fixed circular grid.

Readings (the pages give no bit allocation, grid or codebook):
* d is a power of two; L = log2 d levels.  Level 1 pairs (y_2i, y_2i+1):
  r = hypot, theta = atan2(y_2i+1, y_2i) taken in [0, 2 pi).  Level l >= 2
  pairs the radii of level l - 1: theta = atan2(r_2i+1, r_2i) in [0, pi/2].
  The final radius is ||y|| = ||x||, stored as float32 like TurboQuant's norm.
* After a Haar rotation y / ||y|| is uniform on the sphere, so a level-1 angle
  is uniform on the circle, and for l >= 2 (each side of the pair aggregating
  m = 2^(l-1) coordinates) sin^2(theta) ~ Beta(m/2, m/2):
  f_l(theta) = 2 sin^(m-1)(theta) cos^(m-1)(theta) / B(m/2, m/2) on [0, pi/2].
* Level-1 angles take b1 bits on the uniform grid (cell k = [k, k+1) 2 pi / 2^b1,
  centroid at the middle: the Lloyd-Max quantizer of the uniform law);
  levels l >= 2 take bh bits, Lloyd-Max for f_l (thresholds = midpoints,
  a value on a threshold takes the upper cell).  b1 = 4, bh = 2 spends
  (4 d/2 + 2 (d/2 - 1)) / d ~ 3 bits per coordinate.
* Reconstruction runs the tree back down from the stored radius with the
  centroid angles, then x_hat = Pi^T y_hat.
* Packing: the d/2 level-1 codes in the b1-bit layout of TurboQuant's codes
  (as if they were d/2 coordinates), then the d/2 - 1 higher-level codes,
  level 2 first, in the bh-bit layout.
"""
from __future__ import annotations

import math

import numpy as np
from scipy import integrate, special

from .turboquant import code_words, pack_codes_vec, quantize_indices, unpack_codes

TWO_PI = 2.0 * math.pi


def levels(d: int) -> int:
    L = int(round(math.log2(d)))
    if 2 ** L != d or d < 2:
        raise ValueError("PolarQuant needs d a power of two, d >= 2")
    return L


def polar_transform(y: np.ndarray):
    """(R [N], [theta_1 [N, d/2], theta_2 [N, d/4], ..., theta_L [N, 1]])."""
    y = np.atleast_2d(np.asarray(y, dtype=np.float64))
    levels(y.shape[1])
    a, b = y[:, 0::2], y[:, 1::2]
    thetas = [np.mod(np.arctan2(b, a), TWO_PI)]
    r = np.hypot(a, b)
    while r.shape[1] > 1:
        a, b = r[:, 0::2], r[:, 1::2]
        thetas.append(np.arctan2(b, a))
        r = np.hypot(a, b)
    return r[:, 0], thetas


def polar_inverse(R: np.ndarray, thetas) -> np.ndarray:
    """The tree run back down: the inverse of polar_transform."""
    r = np.asarray(R, dtype=np.float64)[:, None]
    for th in reversed(thetas[1:]):
        out = np.empty((r.shape[0], 2 * r.shape[1]))
        out[:, 0::2] = r * np.cos(th)
        out[:, 1::2] = r * np.sin(th)
        r = out
    th = thetas[0]
    y = np.empty((r.shape[0], 2 * r.shape[1]))
    y[:, 0::2] = r * np.cos(th)
    y[:, 1::2] = r * np.sin(th)
    return y


def angle_pdf(theta, level: int):
    """Density of a level-l angle of a uniform point on the sphere."""
    theta = np.asarray(theta, dtype=np.float64)
    if level == 1:
        return np.where((theta >= 0) & (theta < TWO_PI), 1.0 / TWO_PI, 0.0)
    m = 2 ** (level - 1)
    val = 2.0 * np.sin(theta) ** (m - 1) * np.cos(theta) ** (m - 1) / special.beta(m / 2, m / 2)
    return np.where((theta >= 0) & (theta <= math.pi / 2), val, 0.0)


def angle_cdf(theta, level: int):
    theta = np.asarray(theta, dtype=np.float64)
    if level == 1:
        return np.clip(theta / TWO_PI, 0.0, 1.0)
    m = 2 ** (level - 1)
    t = np.clip(theta, 0.0, math.pi / 2)
    return special.betainc(m / 2, m / 2, np.sin(t) ** 2)


def angle_codebook(b: int, level: int, iters: int = 400):
    """(centroids [2^b] ascending, thresholds [2^b - 1]) of a level's angle
    quantizer: the uniform grid on the circle for level 1, Lloyd-Max for f_l
    (conditional means by adaptive quadrature) for l >= 2."""
    K = 2 ** b
    if level == 1:
        c = (np.arange(K) + 0.5) * TWO_PI / K
        return c, np.arange(1, K) * TWO_PI / K
    m = 2 ** (level - 1)
    sd = 0.5 / math.sqrt(m)              # spread of the law around pi/4
    q = np.linspace(-2.0, 2.0, K) if K > 1 else np.zeros(1)
    c = np.clip(math.pi / 4 + sd * q, 1e-6, math.pi / 2 - 1e-6)
    for _ in range(iters):
        t = 0.5 * (c[1:] + c[:-1])
        edges = np.concatenate([[0.0], t, [math.pi / 2]])
        new = np.empty(K)
        for k in range(K):
            lo, hi = edges[k], edges[k + 1]
            mass = angle_cdf(hi, level) - angle_cdf(lo, level)
            mom = integrate.quad(lambda x: x * angle_pdf(x, level), lo, hi, limit=200, epsabs=0, epsrel=1e-13)[0]
            new[k] = mom / mass if mass > 0 else 0.5 * (lo + hi)
        if np.max(np.abs(new - c)) < 1e-15:
            c = new
            break
        c = new
    return c, 0.5 * (c[1:] + c[:-1])


def make_books(d: int, b1: int, bh: int):
    """Codebooks of every level: [(centroids, thresholds)] for l = 1..L."""
    return [angle_codebook(b1 if l == 1 else bh, l) for l in range(1, levels(d) + 1)]


def quant_polar(x: np.ndarray, Pi: np.ndarray, books):
    """PolarQuant of the rows of x: n = ||x|| (float32 as stored), y = Pi x,
    the angle tree of y, every angle's cell against its level's thresholds.
    Returns dict(codes=[per level int64 arrays], norms, thetas, y)."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    y = x @ Pi.T
    R, thetas = polar_transform(y)
    codes = [quantize_indices(th, books[l][1]) for l, th in enumerate(thetas)]
    return dict(codes=codes, norms=np.sqrt(np.sum(x * x, axis=1)).astype(np.float32), thetas=thetas, y=y)


def dequant_polar(codes, norms, Pi, books) -> np.ndarray:
    """x_hat = Pi^T y_hat, y_hat from the stored norm and the centroid angles."""
    thetas = [np.asarray(books[l][0])[np.asarray(c)] for l, c in enumerate(codes)]
    y_hat = polar_inverse(np.asarray(norms, dtype=np.float64), thetas)
    return y_hat @ Pi


def polar_words(d: int, b1: int, bh: int) -> int:
    """uint32 words per vector of the packed PolarQuant codes."""
    return code_words(b1, d // 2) + (code_words(bh, d // 2 - 1) if d > 2 else 0)


def pack_polar(codes, b1: int, bh: int) -> np.ndarray:
    """Level-1 codes in the b1-bit layout over d/2 entries, then levels 2..L
    concatenated (level 2 first) in the bh-bit layout over d/2 - 1 entries."""
    first = pack_codes_vec(codes[0], b1)
    if len(codes) == 1:
        return first
    rest = pack_codes_vec(np.concatenate([np.atleast_2d(c) for c in codes[1:]], axis=1), bh)
    return np.concatenate([first, rest], axis=1)


def unpack_polar(words: np.ndarray, d: int, b1: int, bh: int):
    words = np.atleast_2d(np.asarray(words, dtype=np.uint32))
    w1 = code_words(b1, d // 2)
    codes = [unpack_codes(words[:, :w1], b1, d // 2)]
    if d > 2:
        rest = unpack_codes(words[:, w1:], bh, d // 2 - 1)
        off = 0
        for l in range(2, levels(d) + 1):
            k = d >> l
            codes.append(rest[:, off:off + k])
            off += k
    return codes


def polar_band(y: np.ndarray, books, d: int, tol: float = 1e-5):
    """Masks [per level] of the angles whose cell a float32 evaluation may
    legitimately pick differently: moving the angle to its nearest decision
    boundary displaces the pair it describes (radius r, unit frame y / ||y||)
    by at most tol / sqrt(d) -- the coordinate band of TurboQuant's codes.
    Level-1 boundaries include 0 = 2 pi."""
    y = np.atleast_2d(np.asarray(y, dtype=np.float64))
    n = np.linalg.norm(y, axis=1)
    yu = y / np.where(n > 0, n, 1.0)[:, None]
    _, thetas = polar_transform(yu)
    masks = []
    r = np.hypot(yu[:, 0::2], yu[:, 1::2])
    for l, th in enumerate(thetas, start=1):
        if l > 1:
            r = np.hypot(r[:, 0::2], r[:, 1::2])
        t = np.asarray(books[l - 1][1])
        bounds = np.concatenate([[0.0], t, [TWO_PI]]) if l == 1 else t
        gap = np.min(np.abs(th[..., None] - bounds[None, None, :]), axis=-1)
        masks.append(gap * r <= tol / math.sqrt(d))
    return masks

"""Pins of the float64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a closed
form, a textbook table, brute force on tiny inputs, an invariant, or an
exact moment (mean and variance) over seeded random draws.  Planted mistakes
(a dropped term, a wrong sign, a transposed rotation) fail at least one.
"""
import math
import os

import numpy as np
import pytest
from scipy import integrate, special

import synth
from oracle import codebook as cb
from oracle import turboquant as tq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------- rotation

@pytest.mark.parametrize("d", [3, 8, 64, 128, 200])
def test_rotation_orthogonal_and_haar_signs(d):
    G = synth.gaussian_matrix(d, d, 0, synth.ROT_K)
    Pi = tq.haar_rotation(G)
    I = np.eye(d)
    assert np.max(np.abs(Pi.T @ Pi - I)) < 1e-12
    assert np.max(np.abs(Pi @ Pi.T - I)) < 1e-12
    # G = Pi R with R upper triangular and a positive diagonal (the Haar sign fix)
    R = Pi.T @ G
    assert np.max(np.abs(np.tril(R, -1))) < 1e-10 * np.max(np.abs(R))
    assert np.all(np.diag(R) > 0)


# --------------------------------------------------------------------- coordinate law

@pytest.mark.parametrize("d", [3, 5, 16, 128, 1536])
def test_coordinate_law_normalised_with_variance_one_over_d(d):
    # a uniform point on the unit sphere has E[x_j^2] = 1/d: pins the exponent (d-3)/2
    mass = integrate.quad(lambda x: cb.coord_pdf(x, d), -1, 1, points=[0.0], limit=200)[0]
    var = integrate.quad(lambda x: x * x * cb.coord_pdf(x, d), -1, 1, points=[0.0], limit=200)[0]
    assert abs(mass - 1) < 1e-9
    assert abs(var * d - 1) < 1e-8


def test_coordinate_law_matches_sphere_samples():
    d = 7
    z = synth.rng(3, 99).standard_normal((200000, d))
    x = (z / np.linalg.norm(z, axis=1, keepdims=True))[:, 0]
    for t in (-0.6, -0.2, 0.0, 0.3, 0.7):
        emp = np.mean(x <= t)
        assert abs(emp - cb.coord_cdf(t, d)) < 4 * math.sqrt(0.25 / len(x))


@pytest.mark.parametrize("d", [4, 64, 1536])
def test_cdf_and_first_moment_match_quadrature(d):
    for lo, hi in [(-0.3, -0.01), (-0.02, 0.05), (0.001, 0.2)]:
        m0 = integrate.quad(lambda x: cb.coord_pdf(x, d), lo, hi, limit=200, epsabs=0)[0]
        m1 = integrate.quad(lambda x: x * cb.coord_pdf(x, d), lo, hi, limit=200, epsabs=0)[0]
        assert abs(cb.coord_cdf(hi, d) - cb.coord_cdf(lo, d) - m0) < 1e-11
        assert abs(cb.bin_first_moment(lo, hi, d) - m1) < 1e-11


# --------------------------------------------------------------------- codebook

@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_codebook_d3_is_uniform_quantizer(b):
    # d = 3: f is uniform on [-1, 1]; Lloyd-Max is the uniform quantizer and D = 4^-b
    c, t = cb.lloyd_max(b, 3)
    K = 2 ** b
    expect = (2 * np.arange(K) + 1) / K - 1
    assert np.max(np.abs(c - expect)) < 1e-13
    assert abs(cb.distortion(c, 3) - 4.0 ** -b) < 1e-13


@pytest.mark.parametrize("d", [3, 4, 16, 128, 200, 1536])
def test_codebook_b1_closed_form(d):
    c, t = cb.lloyd_max(1, d)
    e = cb.b1_centroid(d)
    assert abs(c[1] - e) < 1e-13 and abs(c[0] + e) < 1e-13
    assert t[0] == 0.0


def test_b1_centroid_value_d128():
    # Gamma(64) / (sqrt(pi) Gamma(64.5)), evaluated independently at 30 digits
    import mpmath
    with mpmath.workdps(30):
        v = float(mpmath.gamma(64) / (mpmath.sqrt(mpmath.pi) * mpmath.gamma(mpmath.mpf(129) / 2)))
    assert abs(cb.b1_centroid(128) - v) < 1e-15
    assert abs(v - 0.0706616) < 1e-7


@pytest.mark.parametrize("b,d", [(b, d) for b in (1, 2, 3, 4) for d in (8, 64, 128, 200, 1536)])
def test_codebook_symmetric_sorted_and_two_routes_agree(b, d):
    c, t = cb.lloyd_max(b, d)
    c2, t2 = cb.lloyd_max_quadrature(b, d)
    assert np.array_equal(c, -c[::-1])
    assert np.all(np.diff(c) > 0)
    assert np.allclose(t, 0.5 * (c[1:] + c[:-1]), rtol=0, atol=1e-17)
    assert np.max(np.abs(c - c2) / np.abs(c)) < 1e-12


def _max_table():
    rows = {}
    with open(os.path.join(GOLDEN, "gaussian_lloyd_max.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            b = int(parts[0])
            levels = np.array([float(v) for v in parts[1:-1]])
            rows[b] = (levels, float(parts[-1]))
    return rows


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_codebook_large_d_tends_to_gaussian_lloyd_max(b):
    levels, mse = _max_table()[b]
    errs = []
    for d in (200, 1536, 8192):
        c, _ = cb.lloyd_max(b, d)
        pos = c[2 ** (b - 1):] * math.sqrt(d)
        errs.append(np.max(np.abs(pos - levels) / levels))
    assert errs[0] > errs[1] > errs[2] or errs[2] < 5e-4
    assert errs[2] < 2e-3
    # distortion per coordinate tends to Max's MSE for a unit Gaussian
    c, _ = cb.lloyd_max(b, 8192)
    assert abs(cb.distortion(c, 8192) / mse - 1) < 5e-3


@pytest.mark.parametrize("d", [8, 64, 128, 200, 1536])
def test_distortion_between_lower_bound_and_paper_bound(d):
    # lower bound 4^-b; the page's "about 2.7x the bound" read as the upper
    # envelope sqrt(3)*pi/2 * 4^-b ~= 2.72 * 4^-b; D decreases with b
    prev = 1.0
    for b in (1, 2, 3, 4):
        c, _ = cb.lloyd_max(b, d)
        D = cb.distortion(c, d)
        assert 4.0 ** -b <= D <= math.sqrt(3) * math.pi / 2 * 4.0 ** -b
        assert D < prev
        prev = D


def test_distortion_d128_b2_value():
    c, _ = cb.lloyd_max(2, 128)
    assert abs(cb.distortion(c, 128) - 0.11600) < 1e-4


# --------------------------------------------------------------------- quantizer

@pytest.mark.parametrize("d", [3, 4, 5, 8])
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_threshold_count_equals_bruteforce_nearest(d, b):
    c, t = cb.lloyd_max(b, d)
    y = synth.rng(b, d).uniform(-1, 1, 4000)
    y = np.concatenate([y, [-1.0, 1.0], t + 1e-15, t - 1e-15])
    assert np.array_equal(tq.quantize_indices(y, t), tq.nearest_centroid_bruteforce(y, c))
    # a value exactly on a threshold takes the upper cell
    assert np.array_equal(tq.quantize_indices(t, t), np.arange(1, 2 ** b))


@pytest.mark.parametrize("d", [128, 1536])
def test_near_threshold_band_is_one_e_minus_5_over_sqrt_d(d):
    # The parity rule excuses a code only where the rotated unit-frame value lies
    # within 1e-5/sqrt(d) of a decision threshold.  Hand-placed values just inside
    # and just outside the band of every threshold of a real codebook, one exactly
    # on the band edge (the rule is "<="), and values on the centroids (far from
    # every threshold) pin the scale (tol/sqrt(d), not tol*sqrt(d) or tol), the
    # comparison and the reference points (thresholds, not centroids).
    c, t = cb.lloyd_max(3, d)
    w = 1e-5 / math.sqrt(d)
    inside = np.concatenate([t + 0.99 * w, t - 0.99 * w])
    outside = np.concatenate([t + 1.01 * w, t - 1.01 * w])
    assert np.all(tq.near_threshold_mask(inside, t, d))
    assert not np.any(tq.near_threshold_mask(outside, t, d))
    assert not np.any(tq.near_threshold_mask(c, t, d))
    assert np.all(tq.near_threshold_mask(t, t, d))
    # exact band edge: thresholds (0, 0.25) and y = w are represented exactly
    edge = np.array([w, 0.25 + 2 * w, -w])
    assert np.array_equal(tq.near_threshold_mask(edge, np.array([0.0, 0.25]), d), [True, False, True])
    # the mask keeps the shape of its input and decides each coordinate on its own
    y = np.array([[t[0] + 0.5 * w, c[0]], [c[7], t[6] - 2 * w]])
    assert np.array_equal(tq.near_threshold_mask(y, t, d), [[True, False], [False, False]])


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_empirical_mse_matches_closed_form(b):
    d, n = 128, 20000
    Pi = tq.haar_rotation(synth.gaussian_matrix(d, d, 1, synth.ROT_K))
    c, t = cb.lloyd_max(b, d)
    x = synth.unit_rows(n, d, 5)
    idx, norms, y = tq.quant_mse(x, Pi, t)
    per = np.sum((y - c[idx]) ** 2, axis=1)
    D = cb.distortion(c, d)
    assert abs(per.mean() - D) < 4 * per.std() / math.sqrt(n)
    # the dequantized vector carries the same error in the original frame
    xh = tq.dequant_mse(idx, norms, Pi, c)
    rel = np.sum((x - xh) ** 2, axis=1)
    assert abs(rel.mean() - D) < 4 * rel.std() / math.sqrt(n) + 1e-6


def test_rotation_orientation_and_norm_scaling():
    # x = n * Pi^T y0 (y0 a unit vector) must give back y = y0 and the norm n;
    # dequantizing idx with unit norm and rotating forward gives c[idx]:
    # pins y = Pi x (not Pi^T x) and the rescaling by the stored norm
    d, b = 64, 3
    Pi = tq.haar_rotation(synth.gaussian_matrix(d, d, 2, synth.ROT_K))
    c, t = cb.lloyd_max(b, d)
    y0 = synth.unit_rows(50, d, 8)
    n = synth.rng(2, 7).uniform(0.5, 30.0, size=50)
    x = (y0 @ Pi) * n[:, None]
    idx, norms, y = tq.quant_mse(x, Pi, t)
    assert np.max(np.abs(y - y0)) < 1e-13
    assert np.allclose(norms, n.astype(np.float32), rtol=1e-7)
    assert np.array_equal(idx, tq.quantize_indices(y0, t))
    xh = tq.dequant_mse(idx, np.ones(50), Pi, c)
    assert np.max(np.abs(xh @ Pi.T - c[idx])) < 1e-13
    xh = tq.dequant_mse(idx, norms, Pi, c)
    assert np.allclose(xh, (c[idx] @ Pi) * norms.astype(np.float64)[:, None], rtol=0, atol=1e-12)


def test_zero_vector_reading():
    d, b = 32, 2
    Pi = tq.haar_rotation(synth.gaussian_matrix(d, d, 0, synth.ROT_K))
    c, t = cb.lloyd_max(b, d)
    idx, n, y = tq.quant_mse(np.zeros((1, d)), Pi, t)
    assert n[0] == 0 and np.all(idx == tq.quantize_indices(0.0, t))
    assert np.all(tq.dequant_mse(idx, n, Pi, c) == 0)


def test_one_bit_mse_inner_product_bias_is_two_over_pi():
    # E<q, x_hat> = (1 - D) <q, x>; at b = 1, 1 - D = d c^2 -> 2/pi (the page's
    # "1-bit underestimates by 36%")
    for d in (128, 1536, 16384):
        c, _ = cb.lloyd_max(1, d)
        assert abs((1 - cb.distortion(c, d)) - d * c[1] ** 2) < 1e-12
    c, _ = cb.lloyd_max(1, 16384)
    assert abs(16384 * c[1] ** 2 - 2 / math.pi) < 1e-4
    assert abs(1 - 2 / math.pi - 0.3634) < 1e-3
    # regression slope of <q, x_hat> on <q, x> over random x, q, fixed Pi
    d, n = 128, 40000
    Pi = tq.haar_rotation(synth.gaussian_matrix(d, d, 3, synth.ROT_K))
    c, t = cb.lloyd_max(1, d)
    x = synth.unit_rows(n, d, 11)
    q = synth.unit_rows(n, d, 12)
    idx, norms, _ = tq.quant_mse(x, Pi, t)
    xh = tq.dequant_mse(idx, norms, Pi, c)
    a = np.sum(q * x, axis=1)
    e = np.sum(q * xh, axis=1)
    slope = np.sum(a * e) / np.sum(a * a)
    expect = 1 - cb.distortion(c, d)
    resid = e - expect * a
    se = math.sqrt(np.sum((a * resid) ** 2)) / np.sum(a * a)
    assert abs(slope - expect) < 5 * se
    assert abs(slope - 2 / math.pi) < 0.02


@pytest.mark.parametrize("b", [2, 3, 4])
def test_mse_inner_product_shrinks_by_one_minus_distortion(b):
    # The Lloyd centroid condition and the sphere's symmetry give
    # E<q, x_hat> = (1 - D(b, d)) <q, x> at every b (the b = 1 case is the 2/pi
    # above): a wrong centroid, threshold or rotation orientation moves the slope.
    d, n = 128, 40000
    Pi = tq.haar_rotation(synth.gaussian_matrix(d, d, 4, synth.ROT_K))
    c, t = cb.lloyd_max(b, d)
    x = synth.unit_rows(n, d, 21 + b)
    q = synth.unit_rows(n, d, 31 + b)
    idx, norms, _ = tq.quant_mse(x, Pi, t)
    xh = tq.dequant_mse(idx, norms, Pi, c)
    a = np.sum(q * x, axis=1)
    e = np.sum(q * xh, axis=1)
    slope = np.sum(a * e) / np.sum(a * a)
    expect = 1 - cb.distortion(c, d)
    resid = e - expect * a
    se = math.sqrt(np.sum((a * resid) ** 2)) / np.sum(a * a)
    assert abs(slope - expect) < 5 * se
    # and the slope is not 1: the shrinkage is resolved at this sample size
    assert (1 - slope) > 5 * se


# --------------------------------------------------------------------- prod / QJL

@pytest.mark.parametrize("d,b", [(64, 3), (128, 3), (256, 2), (512, 4)])
def test_prod_estimator_unbiased_with_exact_variance(d, b):
    trials = 10000
    Pi = tq.haar_rotation(synth.gaussian_matrix(d, d, 4, synth.ROT_K))
    c, t = cb.lloyd_max(b - 1, d)
    x = synth.scaled_gaussian_rows(1, d, 0.5, seed=21)
    q = synth.gaussian_queries(1, d, seed=22)
    exact = float(q[0] @ x[0])
    errs = np.empty(trials)
    r = None
    for i in range(trials):
        S = synth.gaussian_matrix(d, d, 1000 + i, synth.QJL_K)
        st = tq.quant_prod(x, b, Pi, S, t, c)
        r = st["r"][0]
        errs[i] = tq.prod_estimate(q, st["idx"], st["norms"], st["signs"], st["rnorms"], Pi, S, c, b)[0, 0] - exact
    rn = float(np.float32(np.linalg.norm(r)))
    # the stored residual norm is float32: the estimator is unbiased up to that rounding
    var = ((math.pi / 2) * np.sum(r * r) * np.sum(q * q) - float(q[0] @ r) ** 2) / d
    assert abs(errs.mean()) < 4 * math.sqrt(var / trials) + abs(rn - np.linalg.norm(r)) * 10
    assert abs(errs.var() / var - 1) < 0.06


def test_prod_variance_falls_as_one_over_d():
    vals = []
    for d in (64, 128, 256, 512):
        trials = 4000
        Pi = tq.haar_rotation(synth.gaussian_matrix(d, d, 5, synth.ROT_K))
        c, t = cb.lloyd_max(2, d)
        x = synth.unit_rows(1, d, 31)
        q = synth.unit_rows(1, d, 32)
        errs = []
        for i in range(trials):
            S = synth.gaussian_matrix(d, d, 5000 + i, synth.QJL_K)
            st = tq.quant_prod(x, 3, Pi, S, t, c)
            errs.append(tq.prod_estimate(q, st["idx"], st["norms"], st["signs"], st["rnorms"],
                                         Pi, S, c, 3)[0, 0] - float(q[0] @ x[0]))
        vals.append(d * np.var(errs) / float(np.sum(st["r"] ** 2)))
    # d * Var / ||r||^2 = pi/2 ||q||^2 - <q, r_hat>^2 ~ pi/2 for unit q
    vals = np.array(vals)
    assert np.all(np.abs(vals / (math.pi / 2) - 1) < 0.12)


def test_prod_b1_uses_no_mse_bits_and_sign_zero_is_positive():
    d = 16
    Pi = tq.haar_rotation(synth.gaussian_matrix(d, d, 6, synth.ROT_K))
    S = synth.gaussian_matrix(d, d, 6, synth.QJL_K)
    S[3] = 0.0                                  # (S r)_3 == 0 exactly
    x = synth.gaussian_queries(2, d, seed=6)
    st = tq.quant_prod(x, 1, Pi, S, None, None)
    assert np.all(st["x_hat"] == 0) and np.allclose(st["r"], x)
    assert np.all(st["signs"][:, 3])
    assert np.array_equal(st["signs"], (x @ S.T) >= 0)


# --------------------------------------------------------------------- packing

def _golden_packing():
    cases = []
    with open(os.path.join(GOLDEN, "packing_layout.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            kv = dict(p.split("=", 1) for p in line.split())
            cases.append((int(kv["b"]), [int(v) for v in kv["idx"].split(",")],
                          [int(v, 16) for v in kv["words"].split(",")]))
    return cases


def test_fp16_residual_norm_is_one_rounding_of_the_float64_norm():
    # the stored fp16 norm is the nearest fp16 of ||x - x_hat|| (float64), so it
    # is within half an fp16 ulp (2^-11 relative) of it; everything else equal
    d, b = 64, 3
    Pi = tq.haar_rotation(synth.gaussian_matrix(d, d, 3, synth.ROT_K))
    S = synth.gaussian_matrix(d, d, 3, synth.QJL_K)
    c, t = cb.lloyd_max(b - 1, d)
    x = synth.rng(3, 3).standard_normal((400, d)) * 5
    a = tq.quant_prod(x, b, Pi, S, t, c)
    h = tq.quant_prod(x, b, Pi, S, t, c, rn_dtype=np.float16)
    assert h["rnorms"].dtype == np.float16 and a["rnorms"].dtype == np.float32
    exact = np.sqrt(np.sum((x - a["x_hat"]) ** 2, axis=1))
    rel = np.abs(h["rnorms"].astype(np.float64) - exact) / exact
    assert np.max(rel) <= 2.0 ** -11 and np.max(rel) > 2.0 ** -16
    for k in ("idx", "norms", "signs"):
        assert np.array_equal(a[k], h[k])


@pytest.mark.parametrize("case", _golden_packing())
def test_packing_matches_hand_built_words(case):
    b, idx, words = case
    got = tq.pack_codes(np.array([idx]), b)
    assert [int(w) for w in got[0]] == words
    assert np.array_equal(tq.unpack_codes(got, b, 32)[0], idx)


@pytest.mark.parametrize("b", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("d", [1, 31, 32, 64, 100, 200])
def test_packing_roundtrip_and_padding(b, d):
    idx = synth.rng(b, d).integers(0, 2 ** b, size=(3, d))
    w = tq.pack_codes(idx, b)
    assert w.shape == (3, tq.code_words(b, d)) and w.dtype == np.uint32
    assert np.array_equal(tq.unpack_codes(w, b, d), idx)
    full = tq.unpack_codes(w, b, ((d + 31) // 32) * 32)
    assert np.all(full[:, d:] == 0)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [32, 64, 100, 200])
def test_vectorised_packer_equals_field_by_field_packer(b, d):
    idx = synth.rng(10 + b, d).integers(0, 2 ** b, size=(7, d))
    assert np.array_equal(tq.pack_codes_vec(idx, b), tq.pack_codes(idx, b))


# --------------------------------------------------------------------- attention

def test_attention_uniform_and_dominant_limits():
    B, Hq, Hkv, T, d = 1, 4, 2, 37, 8
    v = synth.rng(0, 1).standard_normal((Hkv, T, d))
    k = synth.rng(0, 2).standard_normal((Hkv, T, d))
    # zero queries: all logits equal -> output is the mean of the values
    q0 = np.zeros((B, Hq, d))
    out, _ = tq.attention_decode(q0, lambda b, h, qs: qs @ k[h].T, lambda b, h: v[h], Hkv)
    for j in range(Hq):
        assert np.allclose(out[0, j], v[j // 2].mean(axis=0), atol=1e-14)
    # a query aligned with one key and a huge scale -> output is that key's value
    q1 = np.zeros((B, Hq, d))
    for j in range(Hq):
        q1[0, j] = k[j // 2][5]
    out, lg = tq.attention_decode(q1, lambda b, h, qs: qs @ k[h].T, lambda b, h: v[h], Hkv, scale=1e4)
    for j in range(Hq):
        assert np.allclose(out[0, j], v[j // 2][np.argmax(k[j // 2] @ k[j // 2][5])], atol=1e-9)
    # weights equal scipy's softmax
    q2 = synth.rng(0, 3).standard_normal((B, Hq, d))
    out, lg = tq.attention_decode(q2, lambda b, h, qs: qs @ k[h].T, lambda b, h: v[h], Hkv)
    p = special.softmax(q2[0, 0] @ k[0].T / math.sqrt(d))
    assert np.allclose(out[0, 0], p @ v[0], atol=1e-13)


def test_prefill_is_causal_softmax_over_each_tokens_visible_keys():
    # every new token's output is scipy's softmax over the keys at or before its
    # position; the last token sees everything (= the decode step), the first
    # one T - nq + 1 keys; a key after a token's position never contributes
    B, nq, Hq, Hkv, T, d = 2, 5, 4, 2, 23, 6
    r = synth.rng(5, 1)
    k = r.standard_normal((B, Hkv, T, d))
    v = r.standard_normal((B, Hkv, T, d))
    q = r.standard_normal((B, nq, Hq, d)) * 2
    est = lambda b, h, rows: rows @ k[b, h].T
    out = tq.attention_prefill(q, est, lambda b, h: v[b, h], Hkv, T)
    for b in range(B):
        for i in range(nq):
            vis = T - nq + i + 1
            for j in range(Hq):
                p = special.softmax(q[b, i, j] @ k[b, j // 2, :vis].T / math.sqrt(d))
                assert np.allclose(out[b, i, j], p @ v[b, j // 2, :vis], atol=1e-13)
    dec, _ = tq.attention_decode(q[:, -1], est, lambda b, h: v[b, h], Hkv)
    assert np.allclose(out[:, -1], dec, atol=1e-13)
    # changing a key after the first token's position leaves that token's output alone
    k2 = k.copy()
    k2[:, :, T - nq + 1:] += 5.0
    out2 = tq.attention_prefill(q, lambda b, h, rows: rows @ k2[b, h].T, lambda b, h: v[b, h], Hkv, T)
    assert np.allclose(out2[:, 0], out[:, 0], atol=1e-13)
    assert not np.allclose(out2[:, -1], out[:, -1])


def test_context_split_softmax_states_merge_to_the_full_softmax():
    # Any split of the context into slices (an empty one included) merges back
    # to scipy's softmax over the whole context; a single slice merges to its
    # own normalised sum; slices of very different logit size still combine
    B, Hq, Hkv, T, d = 2, 4, 2, 50, 6
    r = synth.rng(4, 1)
    k = r.standard_normal((B, Hkv, T, d))
    v = r.standard_normal((B, Hkv, T, d))
    q = r.standard_normal((B, Hq, d)) * 3
    full = np.zeros((B, Hq, d))
    for b in range(B):
        for j in range(Hq):
            p = special.softmax(q[b, j] @ k[b, j // 2].T / math.sqrt(d))
            full[b, j] = p @ v[b, j // 2]
    cuts = [0, 7, 7, 31, 50]   # slices [0,7), [7,7) (empty), [7,31), [31,50)
    parts = [tq.attention_partial(q, lambda b, h, qs, a=a, e=e: qs @ k[b, h, a:e].T,
                                  lambda b, h, a=a, e=e: v[b, h, a:e], Hkv)
             for a, e in zip(cuts[:-1], cuts[1:])]
    ms, ls, accs = (np.stack(x) for x in zip(*parts))
    assert np.all(np.isneginf(ms[1])) and np.all(ls[1] == 0)
    assert np.allclose(tq.merge_attention_partials(ms, ls, accs), full, atol=1e-12)
    one = tq.attention_partial(q, lambda b, h, qs: qs @ k[b, h].T, lambda b, h: v[b, h], Hkv)
    assert np.allclose(tq.merge_attention_partials(*(x[None] for x in one)), full, atol=1e-12)
    out, _ = tq.attention_decode(q, lambda b, h, qs: qs @ k[b, h].T, lambda b, h: v[b, h], Hkv)
    assert np.allclose(out, full, atol=1e-12)
    # a slice whose logits are all far below the others' contributes ~nothing
    ms2 = np.stack([ms[0], ms[2] - 800.0])
    got = tq.merge_attention_partials(ms2, np.stack([ls[0], ls[2]]), np.stack([accs[0], accs[2]]))
    assert np.allclose(got, accs[0] / ls[0][..., None], atol=1e-12)


def test_topk_matches_sorting():
    s = synth.rng(1, 1).standard_normal((5, 300))
    s[0, 10] = s[0, 20] = 9.0                    # tie: lower index first
    i, v = tq.topk(s, 10)
    assert i[0, 0] == 10 and i[0, 1] == 20
    for r in range(5):
        assert np.allclose(v[r], np.sort(s[r])[::-1][:10])


def test_channel_split_takes_largest_scales():
    sc = synth.lognormal_channel_scales(128, 1.0, 0)
    hi, lo = tq.channel_split(sc, 64)
    assert len(hi) == 64 and len(lo) == 64
    assert np.min(sc[hi]) > np.max(sc[lo])
    assert np.array_equal(np.sort(np.concatenate([hi, lo])), np.arange(128))


def test_pack_signs_layout_by_hand():
    """QJL sign bits use the b = 1 code layout of include/tq.h: bit i of word g is
    coordinate 32 g + i, set for a non-negative projection."""
    bits = np.zeros((2, 40), dtype=bool)
    bits[0, [0, 31, 32, 39]] = True
    bits[1, 5] = True
    w = tq.pack_signs(bits)
    assert w.shape == (2, 2)
    assert [int(v) for v in w[0]] == [1 | (1 << 31), 1 | (1 << 7)]
    assert [int(v) for v in w[1]] == [1 << 5, 0]
    assert np.array_equal(tq.unpack_signs(w, 40), bits)
    # a random round trip at a width that leaves a partial last word
    r = synth.rng(0, 99).random((5, 77)) < 0.5
    assert np.array_equal(tq.unpack_signs(tq.pack_signs(r), 77), r)


def test_mse_estimate_by_hand():
    """<q, x_hat> with x_hat = n Pi^T c[idx]: with Pi = I it is n sum_j q_j c[idx_j];
    with a quarter-turn Pi = [[0, 1], [-1, 0]], Pi^T c = (-c_1, c_0)."""
    c = np.array([-1.5, -0.5, 0.5, 1.5])
    est = tq.mse_estimate(np.array([1.0, 2.0, -1.0, 0.5]), np.array([[0, 3, 1, 2]]), np.array([2.0]),
                          np.eye(4), c)
    assert est.shape == (1, 1)
    assert abs(est[0, 0] - 2.0 * (-1.5 + 3.0 + 0.5 + 0.25)) < 1e-12
    Pi = np.array([[0.0, 1.0], [-1.0, 0.0]])
    q = np.array([[3.0, -2.0], [1.0, 1.0]])
    idx = np.array([[0, 1], [1, 1]])
    cc = np.array([0.25, -0.75])
    n = np.array([1.0, 4.0])
    est = tq.mse_estimate(q, idx, n, Pi, cc)
    for i in range(2):
        for k in range(2):
            c0, c1 = cc[idx[k, 0]], cc[idx[k, 1]]
            assert abs(est[i, k] - n[k] * (-q[i, 0] * c1 + q[i, 1] * c0)) < 1e-12

"""Pins of the PolarQuant oracle (oracle/polar.py) against the mathematics:
the polar tree inverts exactly, each level's angle law matches sphere samples
and closed forms, the level-2 one-bit codebook has a closed form, and the
level-1 grid's distortion has a closed form."""
import math

import numpy as np
import pytest
from scipy import integrate

import synth
from oracle import codebook as cb
from oracle import polar as pq
from oracle import turboquant as tq


@pytest.mark.parametrize("d", [2, 4, 8, 128])
def test_polar_tree_inverts_and_keeps_the_norm(d):
    y = synth.rng(1, d).standard_normal((300, d)) * 3
    R, th = pq.polar_transform(y)
    assert np.allclose(R, np.linalg.norm(y, axis=1), rtol=1e-13)
    assert len(th) == pq.levels(d) and [t.shape[1] for t in th] == [d >> l for l in range(1, pq.levels(d) + 1)]
    assert np.all((th[0] >= 0) & (th[0] < 2 * math.pi))
    for t in th[1:]:
        assert np.all((t >= 0) & (t <= math.pi / 2))
    assert np.max(np.abs(pq.polar_inverse(R, th) - y)) < 1e-12


def test_polar_tree_by_hand():
    # y = (3, 4, 0, -5): pairs (3, 4) and (0, -5), radii 5 and 5, top angle pi/4
    R, th = pq.polar_transform(np.array([[3.0, 4.0, 0.0, -5.0]]))
    assert abs(R[0] - math.sqrt(50)) < 1e-14
    assert abs(th[0][0, 0] - math.atan2(4, 3)) < 1e-14
    assert abs(th[0][0, 1] - 1.5 * math.pi) < 1e-14
    assert abs(th[1][0, 0] - math.pi / 4) < 1e-14


@pytest.mark.parametrize("level", [2, 3, 4, 5, 6, 7])
def test_angle_law_normalised_symmetric_and_matches_its_cdf(level):
    mass = integrate.quad(lambda t: pq.angle_pdf(t, level), 0, math.pi / 2, limit=200)[0]
    mean = integrate.quad(lambda t: t * pq.angle_pdf(t, level), 0, math.pi / 2, limit=200)[0]
    assert abs(mass - 1) < 1e-10 and abs(mean - math.pi / 4) < 1e-10
    for a in (0.3, math.pi / 4, 1.1):
        part = integrate.quad(lambda t: pq.angle_pdf(t, level), 0, a, limit=200)[0]
        assert abs(part - pq.angle_cdf(a, level)) < 1e-10


def test_angle_laws_match_rotated_sphere_samples():
    # y = Pi x for Gaussian x: every level's empirical CDF at a few angles
    d, n = 64, 20000
    Pi = tq.haar_rotation(synth.gaussian_matrix(d, d, 2, synth.ROT_K))
    y = synth.rng(2, 2).standard_normal((n, d)) @ Pi.T
    _, th = pq.polar_transform(y)
    for l, t in enumerate(th, start=1):
        vals = t.reshape(-1)
        pts = (0.7, 2.5, 5.0) if l == 1 else (0.5, math.pi / 4, 0.9)
        for a in pts:
            emp = np.mean(vals <= a)
            sd = math.sqrt(0.25 / min(len(vals), n))      # angles of one vector are not independent
            assert abs(emp - pq.angle_cdf(a, l)) < 5 * sd, (l, a)


def test_level2_one_bit_codebook_closed_form():
    # f_2 = sin(2 theta): the split is pi/4 and E[theta | theta < pi/4] = 1/2
    c, t = pq.angle_codebook(1, 2)
    assert abs(t[0] - math.pi / 4) < 1e-12
    assert abs(c[0] - 0.5) < 1e-12 and abs(c[1] - (math.pi / 2 - 0.5)) < 1e-12


@pytest.mark.parametrize("b,level", [(2, 3), (2, 7), (3, 4)])
def test_angle_codebooks_are_lloyd_max_fixed_points(b, level):
    c, t = pq.angle_codebook(b, level)
    assert np.allclose(c, math.pi / 2 - c[::-1], atol=1e-12)            # symmetric about pi/4
    edges = np.concatenate([[0.0], t, [math.pi / 2]])
    for k in range(len(c)):
        mass = pq.angle_cdf(edges[k + 1], level) - pq.angle_cdf(edges[k], level)
        mom = integrate.quad(lambda x: x * pq.angle_pdf(x, level), edges[k], edges[k + 1], limit=200)[0]
        assert abs(mom / mass - c[k]) < 1e-10


@pytest.mark.parametrize("b1", [2, 4])
def test_level1_grid_distortion_closed_form(b1):
    # higher levels exact, level 1 on the uniform grid: a pair of radius r moves
    # by the chord of an error uniform in +-h, h = pi / 2^b1:
    # E ||y - y_hat||^2 = ||y||^2 2 (1 - sin(h) / h)
    d, n = 32, 20000
    y = synth.rng(3, b1).standard_normal((n, d))
    R, th = pq.polar_transform(y)
    c, t = pq.angle_codebook(b1, 1)
    th_hat = [c[tq.quantize_indices(th[0], t)]] + th[1:]
    err = np.sum((pq.polar_inverse(R, th_hat) - y) ** 2, axis=1) / R ** 2
    h = math.pi / 2 ** b1
    assert abs(err.mean() - 2 * (1 - math.sin(h) / h)) < 4 * err.std() / math.sqrt(n)


def test_polar_quant_reconstructs_and_improves_with_bits():
    d, n = 128, 2000
    Pi = tq.haar_rotation(synth.gaussian_matrix(d, d, 4, synth.ROT_K))
    x = synth.scaled_gaussian_rows(n, d, 0.5, seed=4)
    prev = None
    for b1, bh in ((2, 1), (4, 2), (6, 3)):
        books = pq.make_books(d, b1, bh)
        st = pq.quant_polar(x, Pi, books)
        xh = pq.dequant_polar(st["codes"], st["norms"], Pi, books)
        rel = np.mean(np.sum((x - xh) ** 2, axis=1) / np.sum(x * x, axis=1))
        assert prev is None or rel < prev
        prev = rel
        # the stored norm survives exactly: ||x_hat|| = ||x|| (float32)
        assert np.allclose(np.linalg.norm(xh, axis=1), st["norms"], rtol=1e-12)
    # about 3 bits per coordinate at (4, 2); distortion comparable to TurboQuant_mse at 3 bits
    bits = (4 * d // 2 + 2 * (d // 2 - 1)) / d
    assert abs(bits - 3) < 0.05
    books = pq.make_books(d, 4, 2)
    st = pq.quant_polar(x, Pi, books)
    rel = np.mean(np.sum((x - pq.dequant_polar(st["codes"], st["norms"], Pi, books)) ** 2, axis=1) /
                  np.sum(x * x, axis=1))
    c3, _ = cb.lloyd_max(3, d)
    assert rel < 2.5 * cb.distortion(c3, d)


@pytest.mark.parametrize("d", [4, 128, 256])
def test_polar_packing_roundtrip(d):
    books = pq.make_books(d, 4, 2)
    x = synth.rng(5, d).standard_normal((50, d))
    st = pq.quant_polar(x, np.eye(d), books)
    w = pq.pack_polar(st["codes"], 4, 2)
    assert w.shape[1] == pq.polar_words(d, 4, 2)
    back = pq.unpack_polar(w, d, 4, 2)
    for a, b in zip(st["codes"], back):
        assert np.array_equal(a, b)


def test_polar_band_scale_and_reference_points():
    # d = 4: pair radii r0 = 0.6, r1 = 0.8 (unit vector); a level-1 angle just
    # inside / outside tol / (sqrt(d) r0) of a grid boundary, and the level-2
    # angle atan2(0.8, 0.6) moved just inside / outside tol / sqrt(d) (its
    # pair is the whole unit vector) of a level-2 threshold
    d, tol = 4, 1e-5
    books = pq.make_books(d, 4, 2)
    t1 = books[0][1][3]                      # a level-1 boundary, 4 * 2 pi / 16
    t2 = books[1][1][1]                      # the middle level-2 threshold, pi / 4
    w = tol / math.sqrt(d)

    def vec(th0, r0, r1, th1=0.3):
        return np.array([r0 * math.cos(th0), r0 * math.sin(th0), r1 * math.cos(th1), r1 * math.sin(th1)])

    inside = vec(t1 + 0.99 * w / 0.6, 0.6, 0.8)
    outside = vec(t1 + 1.01 * w / 0.6, 0.6, 0.8)
    m_in, m_out = pq.polar_band(inside, books, d), pq.polar_band(outside, books, d)
    assert m_in[0][0, 0] and not m_out[0][0, 0]
    # a boundary at 0 = 2 pi counts too
    assert pq.polar_band(vec(2 * math.pi - 0.5 * w / 0.6, 0.6, 0.8), books, d)[0][0, 0]
    # level 2: angle atan2(r1, r0) = t2 +- just under / over w (the pair radius is 1)
    a_in, a_out = t2 + 0.99 * w, t2 - 1.01 * w
    m_in = pq.polar_band(vec(1.0, math.cos(a_in), math.sin(a_in)), books, d)
    m_out = pq.polar_band(vec(1.0, math.cos(a_out), math.sin(a_out)), books, d)
    assert m_in[1][0, 0] and not m_out[1][0, 0]
    # an angle on a centroid (the middle of its cell) is never excused
    c1 = books[0][0][5]
    assert not pq.polar_band(vec(c1, 0.6, 0.8), books, d)[0][0, 0]

"""Pins of the oracle's Lloyd-Max codebooks and of the stored fp32 tables."""
import math
import os

import numpy as np
import pytest
from scipy import integrate, stats

from oracle import tq_oracle as O
from oracle import gen_codebooks as G


def _beta_sphere_pdf_library(d):
    # Independent density: (x + 1)/2 ~ Beta((D-1)/2, (D-1)/2), from scipy.stats.
    dist = stats.beta((d - 1) / 2.0, (d - 1) / 2.0)
    return lambda x: 0.5 * dist.pdf((x + 1.0) / 2.0)


@pytest.mark.parametrize("d", [16, 64, 128, 256])
def test_beta_density_matches_library(d):
    dens = O.BetaSphereDensity(d)
    ref = _beta_sphere_pdf_library(d)
    xs = np.linspace(-0.9, 0.9, 37)
    np.testing.assert_allclose(dens.pdf(xs), [ref(x) for x in xs], rtol=1e-10, atol=1e-300)
    total, _ = integrate.quad(dens.pdf, -1, 1, points=[0.0], limit=200)
    assert abs(total - 1.0) < 1e-10
    # mass and first moment against numerical integration of the library density
    for lo, hi in [(0.0, 0.05), (0.05, 0.2), (0.2, 1.0)]:
        m0, _ = integrate.quad(ref, lo, hi, epsabs=1e-15, epsrel=1e-12)
        m1, _ = integrate.quad(lambda x: x * ref(x), lo, hi, epsabs=1e-15, epsrel=1e-12)
        assert abs(dens.mass(lo, hi) - m0) < 1e-12
        assert abs(dens.first_moment(lo, hi) - m1) < 1e-12


def test_gaussian_distortions_match_max_1960(golden):
    dens = O.GaussianDensity()
    for bits, value, tol in golden("gaussian_lloyd_max.txt"):
        cb = O.lloyd_max_gaussian(int(bits), 20000)
        dist = O.codebook_distortion(dens, cb)
        assert abs(dist - float(value)) <= float(tol) * float(value), (bits, dist)


def test_gaussian_one_bit_closed_form():
    cb = O.lloyd_max_gaussian(1, 100)
    np.testing.assert_allclose(cb.centroids, [-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)],
                               rtol=1e-14)
    assert abs(O.codebook_distortion(O.GaussianDensity(), cb) - (1 - 2 / math.pi)) < 1e-10


@pytest.mark.parametrize("d", [64, 128, 256])
def test_beta_one_bit_closed_form(d):
    # c = E|x| = Gamma(D/2) / (sqrt(pi) Gamma((D+1)/2)), distortion 1/D - c^2.
    c = math.exp(math.lgamma(d / 2) - 0.5 * math.log(math.pi) - math.lgamma((d + 1) / 2))
    cb = O.lloyd_max_beta(d, 1, 100)
    np.testing.assert_allclose(cb.centroids, [-c, c], rtol=1e-13)
    assert cb.boundaries.tolist() == [0.0]
    dist = O.codebook_distortion(O.BetaSphereDensity(d), cb)
    assert abs(dist - (1.0 / d - c * c)) < 1e-12


@pytest.mark.parametrize("d,bits", [(64, 2), (128, 2), (256, 3), (128, 4)])
def test_lloyd_conditions(d, bits):
    dens = O.BetaSphereDensity(d)
    cb = O.lloyd_max_beta(d, bits, 300_000)
    c, b = cb.centroids, cb.boundaries
    levels = 1 << bits
    assert c.size == levels and b.size == levels - 1
    assert np.all(np.diff(c) > 0) and np.all(np.diff(b) > 0)
    np.testing.assert_array_equal(c, -c[::-1])
    assert b[levels // 2 - 1] == 0.0
    np.testing.assert_array_equal(b, 0.5 * (c[:-1] + c[1:]))
    edges = np.concatenate([[-1.0], b, [1.0]])
    # centroid condition, against the test's own quadrature of the library density
    ref = _beta_sphere_pdf_library(d)
    for i in range(levels // 2, levels):
        m0, _ = integrate.quad(ref, edges[i], edges[i + 1], epsabs=0, epsrel=1e-13, limit=200)
        m1, _ = integrate.quad(lambda x: x * ref(x), edges[i], edges[i + 1], epsabs=0,
                               epsrel=1e-13, limit=200)
        assert abs(c[i] - m1 / m0) < 1e-12


def test_beta_distortion_approaches_gaussian():
    # D * distortion of the Beta-sphere quantizer tends to the N(0,1) value as D grows.
    g = O.codebook_distortion(O.GaussianDensity(), O.lloyd_max_gaussian(2, 2000))
    errs = []
    for d in (64, 128, 256, 1024):
        cb = O.lloyd_max_beta(d, 2, 2000)
        errs.append(abs(d * O.codebook_distortion(O.BetaSphereDensity(d), cb) - g))
    assert errs == sorted(errs, reverse=True)
    assert errs[-1] < 0.002 * g


def _stored(d, bits):
    return G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(d, bits)))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_stored_table_structure(d, bits):
    t = _stored(d, bits)
    levels = 1 << bits
    assert (t.dim, t.bits, t.density_id, t.n_iter) == (d, bits, 0, G.N_ITER)
    assert t.centroids.dtype == np.float32 and t.centroids.size == levels
    assert t.boundaries.size == levels - 1
    np.testing.assert_array_equal(t.centroids, -t.centroids[::-1])
    np.testing.assert_array_equal(t.boundaries, -t.boundaries[::-1])
    assert t.boundaries[levels // 2 - 1] == 0.0
    assert np.all(np.diff(t.centroids) > 0) and np.all(np.diff(t.boundaries) > 0)
    # each boundary lies between its two centroids
    assert np.all(t.centroids[:-1] < t.boundaries) and np.all(t.boundaries < t.centroids[1:])


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_stored_table_centroid_condition(d, bits):
    # The stored fp32 centroids are the conditional means of the library density
    # over the stored fp32 cells, up to fp32 rounding.
    t = _stored(d, bits)
    ref = _beta_sphere_pdf_library(d)
    levels = 1 << bits
    edges = np.concatenate([[-1.0], t.boundaries.astype(np.float64), [1.0]])
    cells = range(levels // 2, levels) if bits <= 6 else range(levels // 2, levels, 5)
    for i in list(cells) + [levels - 1]:
        lo, hi = edges[i], edges[i + 1]
        m0, _ = integrate.quad(ref, lo, hi, epsabs=0, epsrel=1e-12, limit=200)
        m1, _ = integrate.quad(lambda x: x * ref(x), lo, hi, epsabs=0, epsrel=1e-12, limit=200)
        c = float(t.centroids[i])
        tol = 4 * np.spacing(np.float32(c)) + 1e-6 * min(hi - lo, 1.0)
        assert abs(c - m1 / m0) <= tol, (i, c, m1 / m0)


@pytest.mark.parametrize("d,bits", [(64, 1), (128, 1), (256, 1), (64, 2), (128, 2),
                                    (256, 2), (256, 3)])
def test_stored_table_regenerates(d, bits):
    t = _stored(d, bits)
    r = G.build_table(d, bits)
    np.testing.assert_array_equal(t.centroids, r.centroids)
    np.testing.assert_array_equal(t.boundaries, r.boundaries)
    assert t.iterations_run == r.iterations_run


@pytest.mark.parametrize("d", [64, 128, 256])
def test_gaussian_tables_scale_to_max_1960(golden, d):
    # sqrt(D) times the stored N(0, 1/D) table is the N(0, 1) Lloyd-Max quantizer: its
    # distortion under N(0, 1) is Max's (1960) value.
    dens = O.GaussianDensity()
    for bits, value, tol in golden("gaussian_lloyd_max.txt"):
        t = G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(d, int(bits), "gauss")))
        assert t.density_id == 1 and t.dim == d and t.bits == int(bits)
        cb = O.Codebook(centroids=t.centroids.astype(np.float64) * math.sqrt(d),
                        boundaries=t.boundaries.astype(np.float64) * math.sqrt(d),
                        iterations_run=0, n_iter=0)
        dist = O.codebook_distortion(dens, cb)
        assert abs(dist - float(value)) <= float(tol) * float(value), (d, bits, dist)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_gaussian_approximation_approaches_beta_sphere(bits):
    # One coordinate of a uniform unit vector tends to N(0, 1/D): the shipped Gaussian
    # and exact tables, computed from two different densities, agree better as D grows.
    gaps = []
    for d in (64, 128, 256):
        tb = G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(d, bits, "beta")))
        tg = G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(d, bits, "gauss")))
        c_b, c_g = tb.centroids.astype(np.float64), tg.centroids.astype(np.float64)
        gaps.append(np.max(np.abs(c_b - c_g)) / np.max(np.abs(c_b)))
        np.testing.assert_array_equal(tg.centroids, -tg.centroids[::-1])
        assert np.all(np.diff(tg.boundaries) > 0)
    assert gaps[0] > gaps[1] > gaps[2]
    assert gaps[2] < 0.02


@pytest.mark.parametrize("d,bits", [(128, 2), (64, 4)])
def test_gaussian_table_is_the_fp32_of_the_oracle_codebook(d, bits):
    t = G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(d, bits, "gauss")))
    cb = O.lloyd_max_gaussian_dim(d, bits, t.n_iter)
    np.testing.assert_array_equal(t.centroids, cb.centroids.astype(np.float32))
    np.testing.assert_array_equal(t.boundaries, cb.boundaries.astype(np.float32))

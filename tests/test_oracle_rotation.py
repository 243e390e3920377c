"""Pins of the oracle's randomized Hadamard transform."""
import numpy as np
import pytest
import scipy.linalg

from oracle import tq_oracle as O


@pytest.mark.parametrize("d", [1, 2, 4, 64, 128, 256])
def test_hadamard_matches_sylvester_library(d):
    np.testing.assert_array_equal(O.hadamard_matrix(d), scipy.linalg.hadamard(d))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_hadamard_orthogonality_exact(d):
    h = O.hadamard_matrix(d)
    np.testing.assert_array_equal(h @ h.T, d * np.eye(d))


@pytest.mark.parametrize("d", [2, 8, 64, 128, 256])
def test_fwht_equals_explicit_product(d):
    rng = np.random.default_rng(d)
    x = rng.integers(-1000, 1000, size=(5, d)).astype(np.float64)
    np.testing.assert_array_equal(O.fwht(x), x @ scipy.linalg.hadamard(d).T)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_rht_orthogonal(d):
    s = O.rht_signs(d, 0)
    r = O.rht_matrix(d, s)
    assert np.max(np.abs(r.T @ r - np.eye(d))) < 1e-12
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, d))
    y = O.rht_forward(x, s)
    np.testing.assert_allclose(y, x @ r.T, rtol=0, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_allclose(O.rht_inverse(y, s), x, rtol=0, atol=1e-12)


def test_rht_signs_applied_before_transform():
    # e_j maps to s_j * (column j of H) / sqrt(D): the sign multiplies the input.
    d = 64
    s = O.rht_signs(d, 9)
    h = scipy.linalg.hadamard(d)
    for j in (0, 1, 17, 63):
        e = np.zeros(d)
        e[j] = 1.0
        np.testing.assert_allclose(O.rht_forward(e, s), s[j] * h[:, j] / 8.0, atol=0)

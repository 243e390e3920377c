"""Pins of the oracle's randomized Hadamard transform."""
import os

import numpy as np
import torch
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


def _gram_schmidt(g):
    """Modified Gram-Schmidt on the columns of g: Q with R's diagonal positive (the
    unique QR factorisation of that sign convention), written out by loops."""
    d = g.shape[0]
    q = np.array(g, dtype=np.float64, copy=True)
    for j in range(d):
        for i in range(j):
            q[:, j] -= np.dot(q[:, i], q[:, j]) * q[:, i]
        q[:, j] /= np.linalg.norm(q[:, j])
    return q


@pytest.mark.parametrize("d", [16, 64])
def test_haar_matrix_is_orthogonal_and_the_positive_diagonal_qr(d):
    h = O.haar_orthogonal(d, d)
    np.testing.assert_allclose(h.T @ h, np.eye(d), atol=1e-12)
    np.testing.assert_allclose(h @ h.T, np.eye(d), atol=1e-12)
    # the same Gaussian draw, factorised by an independent Gram-Schmidt (R's diagonal
    # positive): the sign fix makes numpy's Householder QR agree with it
    g = np.random.default_rng(d).standard_normal((d, d))
    np.testing.assert_allclose(h, _gram_schmidt(g), atol=1e-10)
    r = h.T @ g
    assert np.all(np.diag(r) > 0) and np.allclose(np.tril(r, -1), 0, atol=1e-10)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(5000) * 10.0 ** rng.integers(-20, 20, 5000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.0078125, 1.01171875]])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(O.bf16_round(x), ref.astype(np.float64))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_shipped_dense_rotation_tables(d):
    from oracle import gen_rotations as GR
    dim, seed, hi, lo = GR.read_table(os.path.join(GR.DEFAULT_OUT, GR.table_filename(d)))
    assert dim == d and seed == d
    rot = O.dense_rotation(d, d)
    np.testing.assert_array_equal(hi, rot.hi)
    np.testing.assert_array_equal(lo, rot.lo)
    # R = hi + lo is within 2^-17 of the Haar matrix entry by entry and exact in fp32
    r = hi + lo
    assert np.all(np.abs(r - rot.haar) <= 2.0 ** -17 * np.abs(rot.haar) + 1e-300)
    np.testing.assert_array_equal(r.astype(np.float32).astype(np.float64), r)
    np.testing.assert_allclose(r.T @ r, np.eye(d), atol=1e-4)


def test_dense_rotation_quantize_and_dequantize():
    d = 128
    rot = O.dense_rotation(d, d)
    from oracle import gen_codebooks as G
    t = G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(d, 4)))
    rng = np.random.default_rng(1)
    x = rng.standard_normal((50, d)) * 2
    idx, n, u, _ = O.quantize_rows(x, rot, t)
    m = rot.hi + rot.lo
    np.testing.assert_allclose(u, (x @ m.T) / np.linalg.norm(x, axis=1, keepdims=True),
                               atol=1e-14)
    xh = O.dequantize_rows(idx, n, t, rot)
    np.testing.assert_allclose(xh, n[:, None].astype(np.float64) * (t.centroids[idx] @ m),
                               atol=1e-12)
    cos = np.sum(x * xh, 1) / np.linalg.norm(x, axis=1) / np.linalg.norm(xh, axis=1)
    assert np.all(cos > 0.99)

"""Pins for the oracle's Hessian and inverse-Hessian diagonal.

Closed forms: H = 2 X^T X of a hand matrix, orthogonal (Hadamard) columns, the
2x2 inverse formula in exact rational arithmetic, diagonal matrices, the
dead-column rule and a non-positive-definite input.
"""
from fractions import Fraction as F

import numpy as np
import pytest
from scipy.linalg import hadamard

from oracle import slim_oracle as O


def test_hessian_hand_3x2():
    X = np.array([[1.0, 2.0], [3.0, 4.0], [5.0, 6.0]])
    # X^T X = [[1+9+25, 2+12+30], [2+12+30, 4+16+36]] = [[35, 44], [44, 56]]
    assert np.array_equal(O.hessian(X), np.array([[70.0, 88.0], [88.0, 112.0]]))


def test_hessian_orthogonal_columns():
    X = hadamard(16)[:, :8].astype(np.float64) * 0.5   # column norms^2 = 16 * 0.25 = 4
    assert np.array_equal(O.hessian(X), 8.0 * np.eye(8))


def test_hessian_chunks_sum():
    rng = np.random.default_rng(5)
    X = rng.integers(-4, 5, size=(64, 6)).astype(np.float64)   # integer data: every sum exact
    assert np.array_equal(O.hessian([X[:10], X[10:40], X[40:]]), O.hessian(X))


def test_hinv_orthogonal_closed_form():
    N, n = 32, 8
    c = np.arange(1, n + 1, dtype=np.float64)
    X = hadamard(N)[:, :n].astype(np.float64) * c        # X^T X = N diag(c^2)
    h = O.hinv_diag(O.hessian(X))
    d = 2.0 * N * c ** 2
    damp = 0.01 * d.mean()
    np.testing.assert_allclose(h, 1.0 / (d + damp), rtol=1e-13)


def test_hinv_2x2_exact():
    H = np.array([[70.0, 88.0], [88.0, 112.0]])
    a, b, c = F(70), F(88), F(112)
    damp = F(1, 100) * (a + c) / 2
    det = (a + damp) * (c + damp) - b * b
    expect = [float((c + damp) / det), float((a + damp) / det)]
    np.testing.assert_allclose(O.hinv_diag(H), expect, rtol=1e-12)


def test_hinv_diagonal_matrix_and_dead_column():
    H = np.diag([4.0, 0.0, 2.0])
    # dead column -> H_11 = 1; mean diag = 7/3; damp = 0.07/3
    d = np.array([4.0, 1.0, 2.0])
    np.testing.assert_allclose(O.hinv_diag(H), 1.0 / (d + 0.07 / 3.0), rtol=1e-14)


def test_not_positive_definite():
    with pytest.raises(O.NotPositiveDefinite):
        O.hinv_diag(np.array([[1.0, 2.0], [2.0, 1.0]]), alpha=0.0)


def test_hinv_properties_random_spd():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((200, 24))
    X[:, 3] *= 25.0
    H = O.hessian(X)
    h = O.hinv_diag(H)
    Hd = O.damped(H)
    # [A^-1]_jj >= 1 / A_jj for SPD A (Cauchy-Schwarz), and equality of A^-1 A = I on the diagonal
    assert np.all(h >= 1.0 / np.diagonal(Hd) * (1 - 1e-12))
    np.testing.assert_allclose(h, np.diagonal(np.linalg.inv(Hd)), rtol=1e-10)

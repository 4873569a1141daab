"""Pins for the oracle's GPTQ backbone (gptq_quantize).

1. A Hessian proportional to the identity makes every row of U zero off the
   diagonal: nothing is compensated and GPTQ reduces to SQC on the original
   weights (codes, scale, zero, tau index all equal sqc_calibrate's).
2. Conditional least squares, the property the compensation is built to
   have: once columns 0..j are fixed to their quantized values q_F, the
   working weights of the remaining columns R minimise the quadratic error
   (w - w0)^T H_d (w - w0) over w_R, i.e.
       w_R = w0_R - H_RR^-1 H_RF (q_F - w0_F),
   solved here with np.linalg.solve on the damped Hessian, row by row, for
   several j (a wrong sign, a transposed U or a wrong row of U breaks it).
3. U really is the upper Cholesky factor of the damped inverse Hessian, and
   the diagonal returned is that inverse's diagonal (checked against the
   rest of the oracle's own inverse-Hessian step, which uses L^-1 instead).
4. Compensation lowers the layer's output error against plain SQC on a
   layer with correlated inputs (the reason GPTQ exists), and codes stay in
   range with the group's allocated bits.
"""
import numpy as np
import pytest

from oracle import slim_oracle as O


def layer(seed=0, m=12, n=64, N=400, corr=0.6):
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((N, n))
    X = Z.copy()
    for j in range(1, n):                      # correlated neighbouring channels
        X[:, j] = corr * X[:, j - 1] + np.sqrt(1 - corr * corr) * Z[:, j]
    X[:, 5] *= 8.0
    W = rng.standard_normal((m, n)) * 0.02
    W[:, 5] *= 6.0
    return W, X


def test_identity_hessian_reduces_to_sqc():
    W, _ = layer(seed=1)
    n = W.shape[1]
    H = 2.0 * 300.0 * np.eye(n)
    bits = [1, 3]
    g = O.gptq_quantize(W, H, bits, 32, 0.1, 50)
    r = O.sqc_calibrate(W, g.h, bits, 32, 0.1, 50)
    assert np.array_equal(g.codes, r.codes)
    assert np.array_equal(g.tau_idx, r.tau_idx)
    assert np.array_equal(g.scale64, r.scale64) and np.array_equal(g.zero64, r.zero64)


@pytest.mark.parametrize("j", [0, 7, 31, 40, 62])
def test_compensation_is_conditional_least_squares(j):
    W, X = layer(seed=2)
    m, n = W.shape
    H = O.hessian(X)
    Hd = O.damped(H)
    g = O.gptq_quantize(W, H, [2, 2], 32, 0.1, 50, snapshot_after=j)
    F, R = np.arange(j + 1), np.arange(j + 1, n)
    for i in range(m):
        dF = g.Wq[i, F] - W[i, F]
        wR = W[i, R] - np.linalg.solve(Hd[np.ix_(R, R)], Hd[np.ix_(R, F)] @ dF) if R.size else W[i, R]
        np.testing.assert_allclose(g.snapshot[i, R], wR, rtol=1e-9, atol=1e-12)


def test_factor_is_the_cholesky_of_the_damped_inverse():
    _, X = layer(seed=3, n=48)
    H = O.hessian(X)
    U, hd = O.gptq_factor(H)
    assert np.allclose(np.tril(U, -1), 0.0)
    assert np.all(np.diagonal(U) > 0)
    np.testing.assert_allclose(U.T @ U, np.linalg.inv(O.damped(H)), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(hd, O.hinv_diag(H), rtol=1e-10)


def test_compensation_lowers_output_error_and_codes_in_range():
    W, X = layer(seed=4, m=24, n=128)
    H = O.hessian(X)
    bits = [3, 2, 2, 1]
    g = O.gptq_quantize(W, H, bits, 32, 0.1, 50)
    r = O.sqc_calibrate(W, O.hinv_diag(H), bits, 32, 0.1, 50)
    Wr = O.dequant_codes(r.codes, r.scale64, r.zero64, 32)
    e_gptq = np.sum((X @ (g.Wq - W).T) ** 2)
    e_sqc = np.sum((X @ (Wr - W).T) ** 2)
    assert e_gptq < 0.8 * e_sqc
    for c, b in enumerate(bits):
        q = g.codes[:, c * 32:(c + 1) * 32]
        assert q.min() >= 0 and q.max() <= 2 ** b - 1
    np.testing.assert_allclose(O.dequant_codes(g.codes, g.scale64, g.zero64, 32), g.Wq, rtol=0, atol=1e-15)

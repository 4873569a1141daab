"""Pins for the min-max quantizer, the 3-sigma mask, the tau grid and SQC.

The 128-element group w_j = -1 + 2j/127 (j < 127) with w_127 = 5 is worked
out by hand below: its mean, sigma (exact rationals), mask, range, scale and
zero-point, and its codes at bits 1, 2, 3 and tau indices 0, 24, 49, via the
threshold form of rounding derived in each comment.
"""
import math
from fractions import Fraction as F

import numpy as np
import pytest

from oracle import slim_oracle as O


def hand_group():
    w = np.array([-1.0 + 2.0 * j / 127.0 for j in range(128)])
    w[127] = 5.0
    return w


def test_hand_group_mask_and_moments():
    wf = [F(-1) + F(2 * j, 127) for j in range(127)] + [F(5)]
    mu = sum(wf) / 128
    assert mu == F(1, 32)                      # sum_{j<127} w_j = -127 + 126 = -1; plus 5 gives 4
    var = sum((x - mu) ** 2 for x in wf) / 128
    sd = math.sqrt(float(var))
    assert float(mu + 3 * F(sd)) < 5.0 and float(mu + 3 * F(sd)) > float(F(125, 127))
    assert float(mu - 3 * F(sd)) < -1.0
    mask = O.salient_mask(hand_group()[None, :])[0]
    assert mask.tolist() == [False] * 127 + [True]


def test_hand_group_minmax():
    w = hand_group()[None, :]
    for b, s0, z0 in ((1, 6.0, 1.0 / 6.0), (2, 2.0, 0.5), (3, 6.0 / 7.0, 7.0 / 6.0)):
        lo, hi, s, z, deg = O.minmax_params(w, b)
        assert lo[0] == -1.0 and hi[0] == 5.0 and not deg[0]
        assert s[0] == pytest.approx(s0, rel=1e-15)
        assert z[0] == pytest.approx(z0, rel=1e-15)


def test_tau_grid():
    t = O.tau_grid(0.1, 50)
    assert t.size == 50
    assert t[0] == pytest.approx(0.9, rel=1e-15) and t[49] == pytest.approx(1.1, rel=1e-15)
    assert t[24] == pytest.approx(0.9 + 0.2 * 24 / 49, rel=1e-15)
    assert not np.any(t == 1.0)                 # 1.0 is not on the 50-point grid
    assert O.tau_grid(0.1, 1).tolist() == [1.0]
    assert O.tau_grid(0.1, 51)[25] == 1.0


def expected_hand_codes(b, tau):
    w = hand_group()
    if b == 1:
        # u = (w/tau + 1)/6; q = 1 iff u > 1/2 iff w > 2 tau
        q = (w > 2 * tau).astype(int)
    elif b == 2:
        # u = w/(2 tau) + 1/2; q = 0 for w < 0, 1 for 0 < w < 2 tau, 2 for 2tau < w < 4 tau, 3 above 4tau
        q = np.where(w < 0, 0, np.where(w < 2 * tau, 1, np.where(w < 4 * tau, 2, 3)))
    else:
        # u = (7/6)(w/tau + 1); u = q - 1/2 (boundary between q-1 and q) at w/tau = (6q - 10)/7
        thr = np.array([(6 * q - 10) / 7.0 for q in range(1, 8)])
        assert np.min(np.abs(w[:, None] / tau - thr[None, :])) > 1e-6
        q = np.sum(w[:, None] / tau > thr[None, :], axis=1)
    return q


@pytest.mark.parametrize("b", [1, 2, 3])
@pytest.mark.parametrize("t", [0, 24, 49])
def test_hand_group_codes(b, t):
    tau = 0.9 + 0.2 * t / 49
    w = hand_group()[None, :]
    lo, hi, s0, z0, _ = O.minmax_params(w, b)
    q, wq = O.fake_quant(w, tau * s0, z0, b)
    exp = expected_hand_codes(b, tau)
    assert q[0].astype(int).tolist() == exp.tolist()
    # the outlier: b=3 at tau=1.1 gives u = (7/6)(5/1.1 + 1) = 6.47 -> 6; else clamps at qmax
    if b == 3 and t == 49:
        assert q[0, 127] == 6
    else:
        assert q[0, 127] == 2 ** b - 1


def test_rint_half_even_and_rtn():
    w = np.array([[0.0, 0.5, 1.5, 3.0]])            # s0 = 1, z0 = 0 at 2 bits
    q, wq = O.fake_quant(w, np.array([1.0]), np.array([0.0]), 2)
    assert q[0].tolist() == [0.0, 0.0, 2.0, 3.0]    # 0.5 -> 0 and 1.5 -> 2 (ties to even)
    Wq = O.rtn_dequant(np.array([[-1.0, 0.5, 1.0, 1.0]]), [1], 4)
    # s0 = 2, z0 = 0.5: u = [0, 0.75, 1, 1] -> q = [0, 1, 1, 1] -> w_hat = 2 (q - 0.5)
    assert Wq[0].tolist() == [-1.0, 1.0, 1.0, 1.0]


def test_degenerate_group_exact():
    W = np.full((2, 8), 0.25)
    W[1] = -3.0
    assert np.array_equal(O.rtn_dequant(W, [2], 8), W)
    r = O.sqc_calibrate(W, np.ones(8), [2], 8, 0.1, 50)
    assert np.all(r.codes == 0) and np.all(r.tau_idx == 0)
    assert np.array_equal(O.dequant_codes(r.codes, r.scale, r.zero, 8), W)


def test_sqc_error_hand():
    w = np.array([[1.0, 2.0, 3.0, 10.0]])
    wq = np.array([[1.0, 2.0, 2.0, 8.0]])
    delta = np.array([[1.0, 1.0, 1.0, 2.0]])
    # delta e^2 = [0, 0, 1, 8]
    E = O.sqc_error(w, delta, np.array([[False, False, False, True]]), wq)
    assert E[0] == pytest.approx(8.0 + 1.0 / 3.0, rel=1e-15)
    E0 = O.sqc_error(w, delta, np.zeros((1, 4), bool), wq)
    assert E0[0] == pytest.approx(9.0 / 4.0, rel=1e-15)


def test_sqc_exact_grid_picks_tau_one():
    rng = np.random.default_rng(1)
    W = rng.integers(0, 4, size=(6, 32)).astype(np.float64)
    W[:, 0], W[:, 1] = 0.0, 3.0                     # every row spans [0, 3]: s0 = 1 at 2 bits
    r = O.sqc_calibrate(W, np.ones(32), [2], 32, 0.1, 51)
    assert np.all(r.tau_idx == 25)                  # tau_25 = 1 reconstructs exactly
    assert np.array_equal(r.codes, W.astype(np.int64))


def test_sqc_lambda_zero_is_rtn():
    rng = np.random.default_rng(2)
    W = rng.standard_normal((8, 64)) * 0.02
    bits = [1, 3]
    r = O.sqc_calibrate(W, np.ones(64) * 0.3, bits, 32, 0.0, 50)
    assert np.all(r.tau_idx == 0)
    np.testing.assert_allclose(O.dequant_codes(r.codes, r.scale64, r.zero64, 32),
                               O.rtn_dequant(W, bits, 32), rtol=0, atol=1e-15)


def test_sqc_outputs_on_grid_and_in_range():
    rng = np.random.default_rng(7)
    W = rng.standard_normal((16, 96)) * 0.02
    W[:, 5] = 0.4
    bits = [1, 2, 3]
    h = rng.uniform(0.1, 1.0, 96)
    r = O.sqc_calibrate(W, h, bits, 32, 0.1, 50)
    for c, b in enumerate(bits):
        q = r.codes[:, c * 32:(c + 1) * 32]
        assert q.min() >= 0 and q.max() <= 2 ** b - 1
    assert np.all((r.tau_idx >= 0) & (r.tau_idx < 50))
    # the chosen error is no larger than tau = first or last grid point's
    taus = O.tau_grid(0.1, 50)
    for c, b in enumerate(bits):
        w = W[:, c * 32:(c + 1) * 32]
        lo, hi, s0, z0, _ = O.minmax_params(w, b)
        d = O.element_salience(w, h[c * 32:(c + 1) * 32])
        mk = O.salient_mask(w)
        best = O.sqc_error(w, d, mk, O.fake_quant(w, taus[r.tau_idx[:, c]] * s0, z0, b)[1])
        for t in (0, 49):
            assert np.all(best <= O.sqc_error(w, d, mk, O.fake_quant(w, taus[t] * s0, z0, b)[1]))
    assert 0.0 < r.mask_rate < 0.05


def test_mask_rate_gaussian_near_two_sided_tail():
    rng = np.random.default_rng(11)
    w = rng.standard_normal((4000, 128))
    rate = O.salient_mask(w).mean()
    assert 0.0015 < rate < 0.0040                   # two-sided 3-sigma tail is 0.27%

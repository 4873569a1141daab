"""Pins for how sqc_calibrate applies the clipping factor tau, and for its tie rule.

SliM-LLM write-up (rkmt.cn), section 组件二 SQC: one quantizer is shared by the
salient and the other weights of a group; its parameters "(tau^s, tau^z)" are
searched over n = 50 candidates tau spread linearly in [1 - lambda, 1 + lambda]
(lambda = 0.1), keeping the least l2 reconstruction error. The reading taken
(clipping) scales the min-max range to [tau lo, tau hi]: s = tau s0 while the
zero-point stays z0 = -lo / s0. The other plausible reading keeps s = tau s0
but also scales the zero, z = tau z0. The tests below tell the two apart.

1. The hand group (w_j = (2j - 127)/127 for j < 127, w_127 = 5) with h_j = 1
   for j < 127 and h_127 = 10, so delta_j = w_j^2 and delta_127 = 1/4. Its mask
   is {127} (see test_oracle_quantizer). For every tau on the grid the codes
   are found by rounding exact rationals (Fraction arithmetic, half to even),
   the error E(tau) = delta_127 e_127^2 + (1/127) sum_{j<127} delta_j e_j^2 is
   summed exactly, and t* is the first minimiser. Worked out this way:
       clipping reading:   t* = 12 (b = 1), 21 (b = 2), 24 (b = 3)
       z = tau z0 reading: t* = 0  (b = 1), 20 (b = 2), 22 (b = 3)
   so a quantizer that scaled the zero-point would fail every case.
2. A dense tau scan. With delta equal for every element and an empty mask the
   loss is the plain mean squared error. Under the clipping reading the
   reconstruction is w_hat(tau) = tau * Q(w / tau), Q the min-max quantizer of
   the unclipped range (s = tau s0, z = z0 turn rint(w/s + z0) into
   rint((w/tau - lo)/s0), and s (q - z0) into tau (lo + s0 q)). That form is
   evaluated on 9997 values of tau whose every 204th point is a grid point;
   the oracle's errors at the grid points and its choice must agree with it.
"""
from fractions import Fraction as F

import numpy as np
import pytest

from oracle import slim_oracle as O

S0_Z0 = {1: (F(6), F(1, 6)), 2: (F(2), F(1, 2)), 3: (F(6, 7), F(7, 6))}   # lo = -1, hi = 5
TAU_NUM = 441                                  # tau_t = (441 + 2t) / 490 = 0.9 + 0.2 t / 49


def _hand():
    wf = [F(2 * j - 127, 127) for j in range(127)] + [F(5)]
    h = np.ones(128)
    h[127] = 10.0
    return wf, h


def _rint_half_even(u: F) -> int:
    q = u.__floor__()
    r = u - q
    if r > F(1, 2) or (r == F(1, 2) and q % 2 == 1):
        q += 1
    return int(q)


def _exact_errors(b, zero_scaled):
    """E(tau_t), t < 50, and the codes, in exact rational arithmetic."""
    wf, _ = _hand()
    s0, z0 = S0_Z0[b]
    qmax = 2 ** b - 1
    d127 = F(5 * 5, 10 * 10)
    errs, codes = [], []
    for t in range(50):
        tau = F(TAU_NUM + 2 * t, 490)
        s = tau * s0
        z = tau * z0 if zero_scaled else z0
        q = [min(max(_rint_half_even(x / s + z), 0), qmax) for x in wf]
        wq = [s * (qi - z) for qi in q]
        e = d127 * (wf[127] - wq[127]) ** 2 + sum(x * x * (x - y) ** 2 for x, y in zip(wf[:127], wq[:127])) / 127
        errs.append(e)
        codes.append(q)
    return errs, codes


def _first_argmin(v):
    best = 0
    for t in range(1, len(v)):
        if v[t] < v[best]:
            best = t
    return best


@pytest.mark.parametrize("b,t_clip,t_zero_scaled", [(1, 12, 0), (2, 21, 20), (3, 24, 22)])
def test_hand_group_tau_choice(b, t_clip, t_zero_scaled):
    errs, codes = _exact_errors(b, zero_scaled=False)
    assert _first_argmin(errs) == t_clip
    assert _first_argmin(_exact_errors(b, zero_scaled=True)[0]) == t_zero_scaled   # the other reading
    wf, h = _hand()
    w = np.array([float(x) for x in wf])[None, :]
    r = O.sqc_calibrate(w, h, [b], 128, 0.1, 50)
    assert r.tau_idx[0, 0] == t_clip
    assert r.codes[0].tolist() == codes[t_clip]
    s0, z0 = S0_Z0[b]
    assert r.scale64[0, 0] == pytest.approx(float(F(TAU_NUM + 2 * t_clip, 490) * s0), rel=1e-15)
    assert r.zero64[0, 0] == pytest.approx(float(z0), rel=1e-15)
    srt = sorted(errs)
    assert r.margin[0, 0] == pytest.approx(float((srt[1] - srt[0]) / srt[0]), rel=1e-9)


def test_hand_group_tie_takes_smallest_index():
    # a group on an exact grid (lo = 0, hi = 3 at 2 bits) with lambda = 0: every
    # candidate is tau = 1 and errors tie exactly, so t* must be 0
    W = np.array([[0.0, 1.0, 2.0, 3.0] * 8])
    r = O.sqc_calibrate(W, np.ones(32), [2], 32, 0.0, 7)
    assert r.tau_idx[0, 0] == 0 and r.margin[0, 0] == 0.0


def _dense_mse(w, b, taus):
    """Mean squared error of w_hat(tau) = tau * Q(w / tau) for each tau (rows of w: groups)."""
    qmax = 2 ** b - 1
    lo = w.min(axis=1, keepdims=True)
    s0 = (w.max(axis=1, keepdims=True) - lo) / qmax
    out = np.empty((w.shape[0], taus.size))
    for i, tau in enumerate(taus):
        q = np.clip(np.rint((w / tau - lo) / s0), 0, qmax)
        out[:, i] = np.mean((w - tau * (lo + s0 * q)) ** 2, axis=1)
    return out


@pytest.mark.parametrize("b", [1, 2, 3])
def test_dense_tau_scan_plain_mse(b):
    rng = np.random.default_rng(100 + b)
    w = rng.uniform(-1.0, 1.0, size=(40, 64))      # uniform: 3 sigma = 1.73 > max |w - mu|, empty mask
    assert not O.salient_mask(w).any()
    dense = 0.9 + 0.2 * np.arange(49 * 204 + 1) / (49 * 204)
    grid_idx = np.arange(50) * 204
    np.testing.assert_allclose(dense[grid_idx], O.tau_grid(0.1, 50), rtol=1e-15)
    mse = _dense_mse(w, b, dense)
    on_grid = mse[:, grid_idx]
    # one row per call, with h = |w| of that row, so delta = w^2 / h^2 = 1 for every element
    rows = [O.sqc_calibrate(w[i:i + 1], np.abs(w[i]), [b], 64, 0.1, 50) for i in range(w.shape[0])]

    class r:  # the rows' results stacked
        tau_idx = np.concatenate([x.tau_idx for x in rows])
        scale64 = np.concatenate([x.scale64 for x in rows])
        zero64 = np.concatenate([x.zero64 for x in rows])
    # the oracle's choice is the grid point of least MSE in the dense scan
    assert r.tau_idx[:, 0].tolist() == np.argmin(on_grid, axis=1).tolist()
    # and its error there equals the scan's value (the weighted loss reduces to MSE)
    lo, hi, s0, z0, _ = O.minmax_params(w, b)
    np.testing.assert_allclose(r.scale64[:, 0], O.tau_grid(0.1, 50)[r.tau_idx[:, 0]] * s0, rtol=1e-15)
    np.testing.assert_allclose(r.zero64[:, 0], z0, rtol=1e-15)
    _, wq = O.fake_quant(w, r.scale64[:, 0], r.zero64[:, 0], b)
    np.testing.assert_allclose(np.mean((w - wq) ** 2, axis=1), on_grid.min(axis=1), rtol=1e-12)
    # the dense minimum is never above the grid minimum, and is close to it
    assert np.all(mse.min(axis=1) <= on_grid.min(axis=1) * (1 + 1e-15))

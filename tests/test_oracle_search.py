"""Pins for the output-KL objective, the balanced allocation and the SBA search.

KL is checked against scipy.stats.entropy and the binary closed form. The
search is checked against brute force: every balanced allocation is built by
hand from per-level dequantized weights and scored with scipy, independently
of sba_search's own loop.
"""
import itertools

import numpy as np
import pytest
from scipy.special import softmax
from scipy.stats import entropy

from oracle import slim_oracle as O
from post_weight_quantization_hessian_b200 import synthetic as syn


def test_kl_matches_scipy_entropy():
    rng = np.random.default_rng(0)
    Y = rng.standard_normal((7, 11)) * 2
    Yq = Y + rng.standard_normal((7, 11)) * 0.3
    ref = [entropy(softmax(Y[t]), softmax(Yq[t])) for t in range(7)]
    np.testing.assert_allclose(O.kl_per_token(Y, Yq), ref, rtol=1e-12)


def test_kl_binary_closed_form_and_invariants():
    a, b = 0.7, -0.4
    p, q = 1 / (1 + np.exp(-a)), 1 / (1 + np.exp(-b))
    exp = p * np.log(p / q) + (1 - p) * np.log((1 - p) / (1 - q))
    got = O.kl_per_token(np.array([[a, 0.0]]), np.array([[b, 0.0]]))[0]
    assert got == pytest.approx(exp, rel=1e-13)
    Y = np.array([[1.0, 2.0, 3.0]])
    assert O.kl_per_token(Y, Y)[0] == 0.0
    assert O.kl_per_token(Y + 5.0, Y - 2.0)[0] == pytest.approx(0.0, abs=1e-15)


def test_allocation_balanced():
    order = np.array([3, 0, 5, 1, 4, 2])
    for p in range(4):
        bits = O.allocation(order, 2, p)
        assert bits.sum() == 12
        assert (bits == 3).sum() == p and (bits == 1).sum() == p
    assert O.allocation(order, 2, 2).tolist() == [3, 2, 1, 3, 1, 2]   # up {3, 0}, down {4, 2}
    with pytest.raises(ValueError):
        O.allocation(order, 2, 4)
    assert O.sba_candidates(32) == 17           # 16 moves after the uniform start


def small_layer(seed=0, m=24, n=48, N=300, g=8):
    spec = syn.LayerSpec(name="t", m=m, n=n, N=N, x_dtype="f32", group=g, avg_bits=2, seed=seed,
                         n_w_salient=3, w_scale=8.0, n_x_outliers=2, x_scale=20.0)
    W = syn.make_weight(spec).astype(np.float64)
    X = syn.activations_f64(spec)
    return W, X


def test_search_matches_brute_force():
    W, X = small_layer()
    g, k = 8, 6
    h = O.hinv_diag(O.hessian(X))
    order = O.salience_order(O.group_salience(W, h, g))
    res = O.sba_search(W, X, order, g, 2)
    # per-level dequantized weights, assembled by hand per allocation
    levels = {b: O.rtn_dequant(W, [b] * k, g) for b in (1, 2, 3)}
    Y = X @ W.T

    def score(bits):
        Wq = np.concatenate([levels[int(b)][:, c * g:(c + 1) * g] for c, b in enumerate(bits)], axis=1)
        Yq = X @ Wq.T
        return np.mean([entropy(softmax(Y[t]), softmax(Yq[t])) for t in range(X.shape[0])])

    brute = []
    for p in range(k // 2 + 1):
        bits = np.full(k, 2)
        bits[order[:p]] = 3
        bits[order[k - p:]] = 1 if p else 2
        brute.append(score(bits))
    np.testing.assert_allclose(res.kl, brute, rtol=1e-10)
    assert res.p_star == int(np.argmin(brute))
    assert res.bits.sum() == 2 * k
    # p = 0 is uniform 2-bit RTN
    assert res.kl[0] == pytest.approx(score([2] * k), rel=1e-12)
    # informational: the salience-ordered restriction vs every balanced allocation
    best_all = min(score(b) for b in itertools.product((1, 2, 3), repeat=k) if sum(b) == 2 * k)
    assert best_all <= res.kl[res.p_star] + 1e-15


def test_reassociation_equals_direct():
    W, X = small_layer(seed=1)
    h = O.hinv_diag(O.hessian(X))
    order = O.salience_order(O.group_salience(W, h, 8))
    a = O.sba_search(W, X, order, 8, 2)
    b = O.sba_search(W, [X[:100], X[100:]], order, 8, 2, reassociate=True)
    np.testing.assert_allclose(a.kl, b.kl, rtol=1e-12, atol=1e-15)
    assert a.p_star == b.p_star


def test_exactly_representable_layer_has_zero_kl():
    rng = np.random.default_rng(9)
    m, g, k = 10, 8, 4
    W = np.empty((m, g * k))
    for i in range(m):
        for c in range(k):
            a, b = rng.standard_normal(2)
            W[i, c * g:(c + 1) * g] = np.where(rng.random(g) < 0.5, a, b)   # two values per group
    X = rng.standard_normal((50, g * k))
    res = O.sba_search(W, X, np.arange(k), g, 2)
    assert np.all(np.abs(res.kl) < 1e-15) and res.p_star == 0


def test_kl_nonnegative_and_high_bits_small():
    W, X = small_layer(seed=2)
    order = np.arange(6)
    lo = O.sba_search(W, X, order, 8, 2).kl
    hi = O.sba_search(W, X, order, 8, 7).kl
    assert np.all(lo >= 0) and np.all(hi >= 0)
    # small-noise KL grows with the output noise variance; 5 more bits divide it by about 4^5
    assert 0.25 / 1024 < hi[0] / lo[0] < 4.0 / 1024


def test_mse_objective_closed_form_through_the_hessian():
    """MSE_p = mean over tokens and outputs of (x (W_p - W)^T)^2
    = trace(E_p (X^T X) E_p^T) / (N m) with E_p = W_p - W: the same number from
    the Gram matrix, without forming any layer output."""
    W, X = small_layer(seed=3)
    g, k = 8, 6
    m, N = W.shape[0], X.shape[0]
    S = O.group_salience(W, O.hinv_diag(O.hessian(X)), g)
    order = O.salience_order(S)
    G = X.T @ X
    for reassociate in (False, True):
        r = O.sba_search(W, X, order, g, 2, reassociate=reassociate, objective="mse")
        for p in range(k // 2 + 1):
            E = O.rtn_dequant(W, O.allocation(order, 2, p), g) - W
            assert r.kl[p] == pytest.approx(np.trace(E @ G @ E.T) / (N * m), rel=1e-10)
        assert r.p_star == int(np.argmin(r.kl))


def test_mse_objective_brute_force_and_bit_growth():
    """Every balanced allocation scored by hand: the search's MSE equals the
    brute-force value for the salience-ordered ones; raising every group's
    bits lowers the error about 4x per bit."""
    W, X = small_layer(seed=4)
    g, k = 8, 6
    order = O.salience_order(O.group_salience(W, O.hinv_diag(O.hessian(X)), g))
    r = O.sba_search(W, X, order, g, 2, objective="mse")
    Y = X @ W.T
    for p in range(k // 2 + 1):
        Yq = X @ O.rtn_dequant(W, O.allocation(order, 2, p), g).T
        assert r.kl[p] == pytest.approx(np.mean((Yq - Y) ** 2), rel=1e-12)
    e = [np.mean((X @ O.rtn_dequant(W, [b] * k, g).T - Y) ** 2) for b in (3, 4, 5, 6)]
    ratios = np.array(e[:-1]) / np.array(e[1:])
    assert np.all((ratios > 2.5) & (ratios < 6.5))


@pytest.mark.parametrize("kind", ["head_tail", "random"])
def test_search_with_a_given_order(kind):
    """Head-tail (groups in position order) and random allocation: the search
    promotes order[:p] and demotes order[k-p:] of the order it is given, and
    its scores equal the brute-force scores of those allocations."""
    W, X = small_layer(seed=5)
    g, k = 8, 6
    order = np.arange(k) if kind == "head_tail" else np.random.default_rng(9).permutation(k)
    for objective in ("kl", "mse"):
        r = O.sba_search(W, X, order, g, 2, objective=objective)
        Y = X @ W.T
        for p in range(k // 2 + 1):
            bits = np.full(k, 2)
            bits[order[:p]] = 3
            if p:
                bits[order[k - p:]] = 1
            Yq = X @ O.rtn_dequant(W, bits, g).T
            ref = (np.mean([entropy(softmax(Y[t]), softmax(Yq[t])) for t in range(X.shape[0])])
                   if objective == "kl" else np.mean((Yq - Y) ** 2))
            assert r.kl[p] == pytest.approx(ref, rel=1e-10)
        assert r.bits.tolist() == O.allocation(order, 2, r.p_star).tolist()

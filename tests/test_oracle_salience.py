"""Pins for the oracle's salience, group means and order."""
import numpy as np

from oracle import slim_oracle as O


def test_hand_4x8():
    W = np.array([[1, 0, 2, 0, 1, 1, 1, 1],
                  [0, 1, 0, 2, 0, 0, 0, 0],
                  [1, 1, 1, 1, 2, 0, 0, 0],
                  [0, 0, 0, 0, 0, 0, 0, 2]], dtype=np.float64)
    h = np.array([1, 1, 2, 2, 1, 2, 1, 2], dtype=np.float64)
    # delta = w^2 / h^2; group 0 sums to 2 + 2 + 2.5 + 0 = 6.5, group 1 to 2.5 + 0 + 4 + 1 = 7.5
    S = O.group_salience(W, h, 4)
    assert S.tolist() == [6.5 / 16, 7.5 / 16]
    assert O.salience_order(S).tolist() == [1, 0]
    d = O.element_salience(W, h)
    assert d[0, 2] == 1.0 and d[2, 2] == 0.25 and d[3, 7] == 1.0


def test_ties_lower_index_first():
    S = np.array([1.0, 3.0, 1.0, 3.0, 2.0])
    assert O.salience_order(S).tolist() == [1, 3, 4, 0, 2]


def test_permutation_equivariance():
    rng = np.random.default_rng(3)
    g, k = 8, 6
    W = rng.standard_normal((5, g * k))
    h = rng.uniform(0.5, 2.0, g * k)
    S = O.group_salience(W, h, g)
    perm = rng.permutation(k)
    cols = np.concatenate([np.arange(c * g, (c + 1) * g) for c in perm])
    S2 = O.group_salience(W[:, cols], h[cols], g)
    np.testing.assert_allclose(S2, S[perm], rtol=1e-14)
    assert perm[O.salience_order(S2)].tolist() == O.salience_order(S).tolist()


def test_scaled_cluster_is_most_salient():
    rng = np.random.default_rng(4)
    W = rng.standard_normal((16, 64)) * 0.02
    W[:, 40:48] *= 6.0
    h = np.ones(64)
    assert O.salience_order(O.group_salience(W, h, 16))[0] == 2

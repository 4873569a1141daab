"""The tolerant comparison helpers of the full-size tests, on hand-made cases."""
import numpy as np
import pytest

from oracle import slim_oracle as O
from parity_util import allocation_ok, comparable_candidates, pstar_ok


def test_comparable_candidates():
    gold = np.arange(8)
    assert comparable_candidates(gold, gold) == [0, 1, 2, 3, 4]
    swapped = np.array([0, 2, 1, 3, 4, 5, 6, 7])       # positions 1 and 2 swapped
    assert comparable_candidates(swapped, gold) == [0, 1, 3, 4]
    tail = np.array([0, 1, 2, 3, 4, 5, 7, 6])          # the two least salient swapped
    assert comparable_candidates(tail, gold) == [0, 2, 3, 4]


def test_allocation_equal_and_pstar_tie():
    order = np.arange(8)
    S = np.linspace(8.0, 1.0, 8)
    kl = np.array([0.5, 0.3, 0.2, 0.20005, 0.4])
    bits = O.allocation(order, 2, 2)
    assert allocation_ok(bits, order, 2, bits, kl, S, 2, 1e-4, 1e-5) == ""
    assert allocation_ok(O.allocation(order, 2, 3), order, 3, bits, kl, S, 2, 1e-4, 1e-5) == "p* (near tie)"
    with pytest.raises(AssertionError):                  # a clear loser
        allocation_ok(O.allocation(order, 2, 1), order, 1, bits, kl, S, 2, 1e-4, 1e-5)


def test_allocation_near_tie_swap():
    gold = np.arange(8)
    S = np.array([8.0, 7.0, 6.0, 6.0 * (1 - 1e-7), 4.0, 3.0, 2.0, 1.0])
    kl = np.array([0.5, 0.3, 0.2, 0.1, 0.4])          # p* = 3 promotes the first three groups
    ref = O.allocation(gold, 2, 3)
    gpu = np.array([0, 1, 3, 2, 4, 5, 6, 7])           # groups 2 and 3 swapped across the boundary
    assert allocation_ok(O.allocation(gpu, 2, 3), gpu, 3, ref, kl, S, 2, 1e-4, 1e-5) == "near-tie swap"
    gpu3 = np.array([0, 3, 2, 1, 4, 5, 6, 7])          # groups 1 and 3 swapped: not a near tie
    with pytest.raises(AssertionError):
        allocation_ok(O.allocation(gpu3, 2, 3), gpu3, 3, ref, kl, S, 2, 1e-4, 1e-5)
    with pytest.raises(AssertionError):                 # bits that are not the GPU order's own allocation
        allocation_ok(ref, gpu3, 3, ref, kl, S, 2, 1e-4, 1e-5)


def test_pstar_tolerance_follows_the_measured_error():
    kl_ref = np.array([0.5, 0.30000, 0.30002, 0.4])
    assert pstar_ok(1, kl_ref, kl_ref + 1e-6)
    # a flip across a 2e-5 gap is accepted only when the run's own error is at least half of it
    assert not pstar_ok(2, kl_ref, kl_ref + np.array([0, 0, 1.1e-5, 0]))
    with pytest.raises(AssertionError):
        pstar_ok(2, kl_ref, kl_ref + np.array([0, 0, 5e-6, 0]))

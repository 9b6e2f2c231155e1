"""Pins of the oracle's index-overlap count (Prism Attention, sec. 3
"Observations", Figure 1 metric): hand cases and brute force over Python
sets, including the edge cases (empty, disjoint, identical, nested)."""
import numpy as np

import oracle


def test_overlap_hand_cases():
    f = oracle.set_overlap
    assert f([1, 3, 5], [3, 4, 5]) == 2
    assert f([], [1, 2]) == 0 and f([1, 2], []) == 0 and f([], []) == 0
    assert f([0, 2, 4, 6], [1, 3, 5, 7]) == 0          # interleaved, disjoint
    assert f([4, 9, 12], [4, 9, 12]) == 3               # identical
    assert f([2, 5], [0, 1, 2, 3, 4, 5, 6]) == 2        # nested
    assert f([7], [7]) == 1 and f([7], [8]) == 0
    assert f([0, 131071], [0, 5, 131071]) == 2          # both ends of a long sequence


def test_overlap_brute_force():
    rng = np.random.default_rng(3)
    for _ in range(300):
        L = int(rng.integers(1, 400))
        na, nb = int(rng.integers(0, L + 1)), int(rng.integers(0, L + 1))
        a = np.sort(rng.choice(L, na, replace=False))
        b = np.sort(rng.choice(L, nb, replace=False))
        assert oracle.set_overlap(a, b) == len(set(a.tolist()) & set(b.tolist()))

"""Pins of the oracle's quantized-selection reading for a proposal layer's own
set (the proposal layer takes the top kappa of its pool by its proposal
scores, no exact rescoring): a hand case, the closed form "top kappa of the
top-kappa_p pool = top kappa of all positions" under one total order, and
brute force with ties."""
import numpy as np

import oracle


def test_pool_topk_hand_case():
    s = np.array([3, 1, 3, 5, 0], np.float32)
    # pool members 0, 2, 3, 4 score 3, 3, 5, 0: position 3, then the tie at 3
    # goes to the lower position 0
    assert oracle.pool_topk(s, [0, 2, 3, 4], 2).tolist() == [0, 3]
    assert oracle.pool_topk(s, [0, 2, 3, 4], 9).tolist() == [0, 2, 3, 4]  # fewer than kappa
    assert oracle.pool_topk(s, [], 3).tolist() == []
    # -0.0 and +0.0 tie: the lower position wins
    z = np.array([-0.0, 0.0, -1.0], np.float32)
    assert oracle.pool_topk(z, [0, 1, 2], 1).tolist() == [0]
    assert oracle.pool_topk(z[::-1].copy(), [0, 1, 2], 1).tolist() == [1]


def test_pool_topk_of_the_proposal_pool_is_the_global_topk():
    rng = np.random.default_rng(8)
    for _ in range(50):
        L = int(rng.integers(1, 3000))
        s = np.round(rng.standard_normal(L) * 4).astype(np.float32)  # many ties
        kp = int(rng.integers(1, L + 1))
        k = int(rng.integers(1, kp + 1))
        pool = oracle.topk_ascending(s, kp)
        assert np.array_equal(oracle.pool_topk(s, pool, k), oracle.topk_ascending(s, k))


def test_pool_topk_brute_force():
    rng = np.random.default_rng(9)
    for _ in range(200):
        L = int(rng.integers(1, 200))
        s = rng.integers(-3, 4, L).astype(np.float32)
        n = int(rng.integers(0, L + 1))
        pool = np.sort(rng.choice(L, n, replace=False)).astype(np.int32)
        k = int(rng.integers(1, 60))
        order = sorted(pool.tolist(), key=lambda t: (-float(s[t]), t))
        want = sorted(order[:min(k, n)])
        assert oracle.pool_topk(s, pool, k).tolist() == want

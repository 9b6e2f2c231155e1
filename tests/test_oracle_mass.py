"""Oracle pins for the softmax-mass group aggregation (a pool member's
selection score is the attention mass the G query heads of its KV head put
on it, each head's softmax over the pool).  The pins use what the
mathematics fixes: a hand-derived case in closed form, the masses summing to
G, a single head reducing to the exact-score order, the large-scale limit
(each head's mass collapsing onto its top member) and brute-force selection."""
import math

import numpy as np
import pytest

import oracle


def _brute(r, pool, k):
    order = sorted(range(len(r)), key=lambda i: (-float(r[i]), i))
    return np.array(sorted(int(pool[i]) for i in order[:min(k, len(r))]), np.int32)


def test_mass_hand_case():
    # head 0: logits 0, 0, 0 (uniform); head 1: 1, 0, 0 at scale 1
    q = np.array([[0, 0], [1, 0]], np.float32)
    K = np.array([[1, 5], [0, 7], [0, -2]], np.float32)
    pool = np.array([0, 1, 2], np.int32)
    r = oracle.refine_scores_mass(q, K, pool, 1.0)
    e = math.e
    want = [1 / 3 + e / (e + 2), 1 / 3 + 1 / (e + 2), 1 / 3 + 1 / (e + 2)]
    assert np.allclose(r, want, rtol=0, atol=1e-15)
    idx, _ = oracle.refine_row_mass(q, K, pool, 2, 1.0)
    assert idx.tolist() == [0, 1]  # members 1 and 2 tie: the lower slot wins


@pytest.mark.parametrize("G", [1, 3, 4, 8])
def test_mass_sums_to_group_size(G):
    rng = np.random.default_rng(10 + G)
    q = rng.standard_normal((G, 64)).astype(np.float32)
    K = rng.standard_normal((900, 64)).astype(np.float32)
    pool = np.sort(rng.choice(900, 333, replace=False)).astype(np.int32)
    r = oracle.refine_scores_mass(q, K, pool, 0.125)
    assert abs(r.sum() - G) < 1e-12 and np.all(r > 0)


def test_single_head_mass_order_is_score_order():
    """exp is increasing, so with one head the mass ranks the members as the
    exact scores do (distinct scores: the sets are equal)."""
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 128)).astype(np.float32)
    K = rng.standard_normal((2000, 128)).astype(np.float32)
    pool = np.sort(rng.choice(2000, 700, replace=False)).astype(np.int32)
    for kap in (1, 50, 699, 700):
        a, _ = oracle.refine_row_mass(q, K, pool, kap, 0.0883883)
        b, _ = oracle.refine_row(q, K, pool, kap)
        assert np.array_equal(a, b), kap


def test_large_scale_mass_goes_to_each_heads_top_member():
    """At a very large scale each head's softmax is one-hot on its top member:
    the masses count, per member, the heads whose top member it is."""
    rng = np.random.default_rng(5)
    G = 6
    q = rng.standard_normal((G, 32)).astype(np.float32)
    K = rng.standard_normal((300, 32)).astype(np.float32)
    pool = np.arange(0, 300, 2, dtype=np.int32)
    r = oracle.refine_scores_mass(q, K, pool, 1e6)
    dots = (K[pool].astype(np.float64) @ q.astype(np.float64).T)  # [n][G]
    tops = dots.argmax(axis=0)
    want = np.bincount(tops, minlength=pool.size).astype(np.float64)
    assert np.allclose(r, want, atol=1e-9)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_mass_selection_is_brute_force(seed):
    rng = np.random.default_rng(seed)
    G, d = 4, 16
    q = rng.integers(-2, 3, (G, d)).astype(np.float32)
    K = rng.integers(-2, 3, (400, d)).astype(np.float32)
    pool = np.sort(rng.choice(400, 150, replace=False)).astype(np.int32)
    r = oracle.refine_scores_mass(q, K, pool, 0.5)
    for kap in (1, 7, 64, 150):
        idx, _ = oracle.refine_row_mass(q, K, pool, kap, 0.5)
        assert np.array_equal(idx, _brute(r, pool, kap)), kap

"""Pins of the oracle's selection-granularity variants: one set per query
head over the group's shared pool, and one pool and set per sequence shared
by every head (the per-KV-head maximum taken over the KV heads as well).
Hand cases, exact integer data ranked by brute force in int64, and the
special cases that reduce to the per-KV-head forms (G = 1, Hkv = 1)."""
import numpy as np

import oracle


def _rank(scores, positions, k):
    order = sorted(range(len(positions)), key=lambda i: (-int(scores[i]), int(positions[i])))
    return sorted(int(positions[i]) for i in order[:k])


def test_heads_hand_case():
    K = np.array([[1, 0], [0, 1], [2, 0], [0, 3]], np.float32)
    q = np.array([[1, 0], [0, 1]], np.float32)
    idx, r = oracle.refine_row_heads(q, K, [0, 1, 2, 3], 1)
    assert idx.tolist() == [[2], [3]]        # each head keeps its own best key
    assert r.tolist() == [[1, 0, 2, 0], [0, 1, 0, 3]]
    idx, _ = oracle.refine_row_heads(q, K, [0, 1, 3], 2)
    assert idx.tolist() == [[0, 1], [1, 3]]  # head 0: 1, then the 0-0 tie to position 1


def test_heads_integer_brute_force():
    rng = np.random.default_rng(21)
    for _ in range(40):
        G, d, L = int(rng.integers(1, 5)), 16, int(rng.integers(1, 300))
        q = rng.integers(-3, 4, (G, d)).astype(np.float32)
        K = rng.integers(-3, 4, (L, d)).astype(np.float32)
        n = int(rng.integers(0, L + 1))
        pool = np.sort(rng.choice(L, n, replace=False)).astype(np.int32)
        k = int(rng.integers(1, 40))
        idx, _ = oracle.refine_row_heads(q, K, pool, k)
        for g in range(G):
            s = (K[pool].astype(np.int64) @ q[g].astype(np.int64)) if n else np.zeros(0, np.int64)
            assert idx[g].tolist() == _rank(s, pool, k)


def test_heads_with_one_head_is_the_group_form():
    rng = np.random.default_rng(22)
    q = rng.standard_normal((1, 64)).astype(np.float32)
    K = rng.standard_normal((500, 64)).astype(np.float32)
    pool = np.sort(rng.choice(500, 300, replace=False)).astype(np.int32)
    idx, r = oracle.refine_row_heads(q, K, pool, 50)
    idx1, r1 = oracle.refine_row(q, K, pool, 50)
    assert np.array_equal(idx[0], idx1) and np.array_equal(r[0], r1)


def test_sequence_hand_case():
    # two KV heads, one query head each: head 0 favours position 1, head 1
    # position 2; the shared score is the maximum over the heads
    q = np.array([[1, 0], [0, 1]], np.float32)
    K = np.array([[[1, 0], [5, 0], [0, 9], [2, 0]],
                  [[0, 1], [0, 0], [0, 4], [0, 3]]], np.float32)
    # position 0: max(1, 1) = 1; 1: max(5, 0) = 5; 2: max(0, 4) = 4; 3: max(2, 3) = 3
    idx, r = oracle.refine_row_seq(q, K, [0, 1, 2, 3], 2)
    assert r.tolist() == [1, 5, 4, 3] and idx.tolist() == [1, 2]
    kq = K.astype(np.int8)
    pool, s = oracle.propose_row_seq(q, kq, np.ones((2, 4), np.float32), 3)
    assert s.tolist() == [1, 5, 4, 3] and pool.tolist() == [1, 2, 3]


def test_sequence_integer_brute_force():
    rng = np.random.default_rng(23)
    for _ in range(30):
        Hkv, G, d, L = int(rng.integers(1, 4)), int(rng.integers(1, 4)), 16, int(rng.integers(1, 200))
        q = rng.integers(-3, 4, (Hkv * G, d)).astype(np.float32)
        kq = rng.integers(-5, 6, (Hkv, L, d)).astype(np.int8)
        kp = int(rng.integers(1, L + 1))
        pool, s = oracle.propose_row_seq(q, kq, np.ones((Hkv, L), np.float32), kp)
        qi = q.astype(np.int64).reshape(Hkv, G, d)
        want = np.max([np.max(kq[h].astype(np.int64) @ qi[h].T, axis=1) for h in range(Hkv)], axis=0)
        assert np.array_equal(s, want.astype(np.float32))
        assert pool.tolist() == _rank(want, np.arange(L), kp)
        K = kq.astype(np.float32)
        k = int(rng.integers(1, kp + 1))
        idx, r = oracle.refine_row_seq(q, K, pool, k)
        assert idx.tolist() == _rank(want[pool], pool, k)


def test_sequence_with_one_kv_head_is_the_group_form():
    rng = np.random.default_rng(24)
    q = rng.standard_normal((4, 64)).astype(np.float32)
    K = rng.standard_normal((1, 700, 64)).astype(np.float32)
    kq, sc = oracle.quantize_rows(K[0])
    pool, s = oracle.propose_row_seq(q, kq[None], sc[None], 200)
    pool1, s1 = oracle.propose_row(q, kq, sc, 200)
    assert np.array_equal(pool, pool1) and np.array_equal(s, s1)
    idx, r = oracle.refine_row_seq(q, K, pool, 60)
    idx1, r1 = oracle.refine_row(q, K[0], pool, 60)
    assert np.array_equal(idx, idx1) and np.array_equal(r, r1)

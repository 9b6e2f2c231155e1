"""Oracle pins for the group-sum selection variant (the G query heads of a KV
head combine by sum instead of max).  Each pin uses something other than the
oracle's own formula: a hand-derived case, exact integer arithmetic checked
in int64, the identity sum_g q_g . k = (sum_g q_g) . k through the maximum
form with one head, and brute-force selection."""
import numpy as np
import pytest

import oracle
from oracle import pipeline


def _brute_topk(scores, k):
    order = sorted(range(len(scores)), key=lambda t: (-float(scores[t]), t))
    return np.array(sorted(order[:min(k, len(scores))]), np.int32)


def test_sum_hand_case():
    # D_0 = q_0 . kq_t = [3, -1, 0], D_1 = q_1 . kq_t = [8, 10, 0]
    q = np.array([[1, 0], [0, 2]], np.float32)
    kq = np.array([[3, 4], [-1, 5], [0, 0]], np.int8)
    scale = np.array([0.5, 2.0, 1.0], np.float32)
    s = oracle.propose_scores(q, kq, scale, agg="sum")
    assert s.tolist() == [5.5, 18.0, 0.0]
    assert oracle.propose_scores(q, kq, scale).tolist() == [4.0, 20.0, 0.0]  # the maximum form
    pool, _ = oracle.propose_row(q, kq, scale, 2, agg="sum")
    assert pool.tolist() == [0, 1]
    pool, _ = oracle.propose_row(q, kq, scale, 1, agg="sum")
    assert pool.tolist() == [1]
    K = np.array([[3, 4], [-1, 5], [0, 0], [1, 1]], np.float32)
    idx, r = oracle.refine_row(q, K, np.array([0, 1, 3], np.int32), 2, agg="sum")
    assert r.tolist() == [11.0, 9.0, 3.0] and idx.tolist() == [0, 1]


def test_single_head_sum_equals_max():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 64)).astype(np.float32)
    kq = rng.integers(-127, 128, (500, 64)).astype(np.int8)
    scale = rng.random(500).astype(np.float32)
    assert np.array_equal(oracle.propose_scores(q, kq, scale, agg="sum"),
                          oracle.propose_scores(q, kq, scale))
    K = rng.standard_normal((300, 64)).astype(np.float32)
    pool = np.arange(0, 300, 3, dtype=np.int32)
    assert np.array_equal(oracle.refine_scores(q, K, pool, agg="sum"), oracle.refine_scores(q, K, pool))


@pytest.mark.parametrize("G", [2, 4, 8])
def test_sum_exact_integer_data(G):
    """Small integers and power-of-two scales keep every sum exact in fp32:
    the scores equal int64 arithmetic and the head-summed query through the
    one-head maximum form; the pools equal brute force (ties: lower position)."""
    rng = np.random.default_rng(G)
    d, L = 32, 700
    q = rng.integers(-3, 4, (G, d)).astype(np.float32)
    kq = rng.integers(-5, 6, (L, d)).astype(np.int8)
    scale = (2.0 ** rng.integers(-4, 3, L)).astype(np.float32)
    exact = (kq.astype(np.int64) @ q.astype(np.int64).T).sum(axis=1) * scale.astype(np.float64)
    s = oracle.propose_scores(q, kq, scale, agg="sum")
    assert np.array_equal(s.astype(np.float64), exact)
    assert np.array_equal(s, oracle.propose_scores(q.sum(axis=0, keepdims=True), kq, scale))
    for k in (1, 50, 333, L, L + 5):
        pool, _ = oracle.propose_row(q, kq, scale, k, agg="sum")
        assert np.array_equal(pool, _brute_topk(exact, k))
    K = rng.integers(-4, 5, (L, d)).astype(np.float32)
    pool = np.sort(rng.choice(L, 400, replace=False)).astype(np.int32)
    rex = (K[pool].astype(np.int64) @ q.astype(np.int64).T).sum(axis=1)
    r = oracle.refine_scores(q, K, pool, agg="sum")
    assert np.array_equal(r.astype(np.int64), rex)
    for k in (1, 100, 400):
        idx, _ = oracle.refine_row(q, K, pool, k, agg="sum")
        assert np.array_equal(idx, pool[_brute_topk(rex, k)])


def test_pipeline_layers_take_the_aggregation():
    rng = np.random.default_rng(9)
    B, Hq, Hkv, d, cu = 2, 8, 2, 32, [0, 300, 520]
    G = Hq // Hkv
    q = rng.standard_normal((B, Hq, d)).astype(np.float32)
    k = rng.standard_normal((Hkv, cu[-1], d)).astype(np.float32)
    kq, sc = pipeline.quantize_layer(k)
    pool, cnt, _ = pipeline.propose_layer(q, kq, sc, cu, 64, agg="sum")
    idx, icnt, _ = pipeline.refine_layer(q, k, cu, pool, cnt, 16, agg="sum")
    for b in range(B):
        for h in range(Hkv):
            qg = q[b, h * G:(h + 1) * G]
            p, _ = oracle.propose_row(qg, kq[h, cu[b]:cu[b + 1]], sc[h, cu[b]:cu[b + 1]], 64, agg="sum")
            assert np.array_equal(pool[b, h, :cnt[b, h]], p)
            i, _ = oracle.refine_row(qg, k[h, cu[b]:cu[b + 1]], p, 16, agg="sum")
            assert np.array_equal(idx[b, h, :icnt[b, h]], i)
    with pytest.raises(ValueError):
        oracle.propose_scores(q[0], kq[0], sc[0], agg="mean")

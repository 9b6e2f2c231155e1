"""Pins of the CPU oracle against what the method and plain mathematics fix.

Nothing here compares the oracle with itself: every expected value comes
from a hand-derived fixture (tests/golden/hand_cases.json), an exact closed
form on integer-valued data, an independent brute force, or a textbook
special case of softmax attention.  Each test is chosen so that a plausible
slip in the oracle -- a dropped scale, sum instead of max over the query
group, a transposed operand, a wrong tie rule, round-half-up instead of
half-even, a lost softmax term -- fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import pipeline

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")))


def _canon(x):
    return float(np.float32(x) + np.float32(0.0))


def _brute_topk(s, k):
    order = sorted(range(len(s)), key=lambda i: (-_canon(s[i]), i))
    return sorted(order[:k])


# ---------------------------------------------------------------- quantize

@pytest.mark.parametrize("case", GOLD["quantize"], ids=lambda c: c["cite"][:30])
def test_quantize_hand_cases(case):
    kq, sc = oracle.quantize_rows(np.array([case["k"]], np.float32))
    assert sc[0] == np.float32(case["scale"])
    assert kq[0].tolist() == case["kq"]


def test_quantize_invariants_random():
    rng = np.random.default_rng(1)
    k = (rng.standard_normal((500, 128)) * rng.uniform(1e-3, 1e3, (500, 1))).astype(np.float32)
    kq, sc = oracle.quantize_rows(k)
    assert np.abs(kq.astype(np.int32)).max() <= 127
    # the element of largest magnitude maps to +-127 with its own sign
    j = np.abs(k).argmax(axis=1)
    top = kq[np.arange(500), j].astype(np.int32)
    assert np.all(np.abs(top) == 127)
    assert np.all(np.sign(top) == np.sign(k[np.arange(500), j]))
    # reconstruction error within half a step (plus fp32 slack)
    err = np.abs(k.astype(np.float64) - sc[:, None].astype(np.float64) * kq)
    assert np.all(err <= sc[:, None] * (0.5 + 1e-5))
    # scale is amax / 127 up to one fp32 rounding
    amax = np.abs(k).max(axis=1).astype(np.float64)
    assert np.allclose(sc, amax / 127.0, rtol=2 ** -23, atol=0)


def test_quantize_power_of_two_rows_exact():
    # k = c * m with integer m (amax 127) and c a power of two: scale = c and
    # the codes reproduce m exactly.
    rng = np.random.default_rng(2)
    m = rng.integers(-127, 128, (64, 32)).astype(np.float32)
    m[:, 5] = 127 * np.where(rng.random(64) < 0.5, 1, -1)
    c = (2.0 ** rng.integers(-20, 20, (64, 1))).astype(np.float32)
    kq, sc = oracle.quantize_rows(m * c)
    assert np.array_equal(sc, c[:, 0])
    assert np.array_equal(kq.astype(np.float32), m)


# ---------------------------------------------------------------- selection

@pytest.mark.parametrize("case", GOLD["select"], ids=lambda c: c["cite"][:30])
def test_select_hand_cases(case):
    assert oracle.topk_ascending(np.array(case["s"], np.float32), case["k"]).tolist() == case["idx"]


def test_select_brute_force_with_ties():
    rng = np.random.default_rng(3)
    vals = np.array([-2.0, -0.0, 0.0, 0.5, 0.5, 1.0, 3.0], np.float32)
    for trial in range(400):
        n = int(rng.integers(1, 48))
        s = rng.choice(vals, n).astype(np.float32)
        k = int(rng.integers(0, n + 3))
        got = oracle.topk_ascending(s, k).tolist()
        assert got == _brute_topk(s, k), (s, k)


def test_select_threshold_property_large():
    rng = np.random.default_rng(4)
    s = rng.standard_normal(20000).astype(np.float32)
    s[::97] = s[5]  # many exact ties at one value
    k = 3000
    got = oracle.topk_ascending(s, k)
    assert got.size == k and np.all(np.diff(got) > 0)
    mask = np.zeros(s.size, bool)
    mask[got] = True
    assert s[mask].min() >= s[~mask].max()
    thr = s[mask].min()
    # at the threshold value the chosen indices all precede the rejected ones
    tie_sel = np.flatnonzero(mask & (s == thr))
    tie_rej = np.flatnonzero(~mask & (s == thr))
    if tie_rej.size:
        assert tie_sel.max() < tie_rej.min()


# ---------------------------------------------------------------- propose

@pytest.mark.parametrize("case", GOLD["propose"], ids=lambda c: c["cite"][:30])
def test_propose_hand_case(case):
    kq, sc = oracle.quantize_rows(np.array(case["k"], np.float32))
    pool, s = oracle.propose_row(np.array(case["q"], np.float32), kq, sc, case["kappa_p"])
    assert s.tolist() == case["scores"]
    assert pool.tolist() == case["pool"]


def test_propose_scores_exact_integer_data():
    # Integer q and codes times power-of-two row scales: every product and
    # partial sum is an exact fp32 value, so the scores must equal the fp64
    # closed form  scale_t * max_g q_g . m_t  exactly.
    rng = np.random.default_rng(5)
    G, d, L = 4, 64, 300
    m = rng.integers(-127, 128, (L, d)).astype(np.float32)
    m[np.arange(L), rng.integers(0, d, L)] = 127.0
    c = (2.0 ** rng.integers(-6, 6, (L, 1))).astype(np.float32)
    q = rng.integers(-8, 9, (G, d)).astype(np.float32)
    kq, sc = oracle.quantize_rows(m * c)
    s = oracle.propose_scores(q, kq, sc)
    want = (c[:, 0].astype(np.float64) * (m.astype(np.float64) @ q.T.astype(np.float64)).max(1))
    assert np.array_equal(s.astype(np.float64), want)
    pool, _ = oracle.propose_row(q, kq, sc, 37)
    assert pool.tolist() == _brute_topk(want, 37)


def test_propose_short_sequence_keeps_everything():
    rng = np.random.default_rng(6)
    kq, sc = oracle.quantize_rows(rng.standard_normal((50, 16)).astype(np.float32))
    pool, _ = oracle.propose_row(rng.standard_normal((2, 16)).astype(np.float32), kq, sc, 64)
    assert pool.tolist() == list(range(50))
    pool, _ = oracle.propose_row(rng.standard_normal((2, 16)).astype(np.float32), kq[:0], sc[:0], 8)
    assert pool.size == 0


# ---------------------------------------------------------------- refine

@pytest.mark.parametrize("case", GOLD["refine"], ids=lambda c: c["cite"][:30])
def test_refine_hand_case(case):
    idx, r = oracle.refine_row(np.array(case["q"], np.float32), np.array(case["K"], np.float32),
                               np.array(case["pool"], np.int32), case["kappa"])
    assert r.tolist() == case["r"]
    assert idx.tolist() == case["idx"]


def test_refine_exact_integer_data_and_subset():
    rng = np.random.default_rng(7)
    G, d, L = 4, 32, 500
    K = rng.integers(-50, 51, (L, d)).astype(np.float32)
    q = rng.integers(-9, 10, (G, d)).astype(np.float32)
    pool = np.sort(rng.choice(L, 120, replace=False)).astype(np.int32)
    idx, r = oracle.refine_row(q, K, pool, 30)
    exact = (K[pool].astype(np.float64) @ q.T.astype(np.float64)).max(1)
    assert np.array_equal(r.astype(np.float64), exact)
    assert idx.tolist() == sorted(pool[_brute_topk(exact, 30)].tolist())
    assert set(idx.tolist()) <= set(pool.tolist())
    # rho = 1: the refined set is the whole pool (static reuse)
    idx1, _ = oracle.refine_row(q, K, pool, pool.size)
    assert np.array_equal(idx1, pool)


def test_refine_over_full_pool_equals_propose_when_codes_are_exact():
    # integer keys with a 127 entry per row: scale = 1 and codes = keys, so
    # the proposal scores are the exact scores and propose(kappa) == refine
    # over the whole context with the same kappa.
    rng = np.random.default_rng(8)
    G, d, L = 4, 64, 400
    K = rng.integers(-127, 128, (L, d)).astype(np.float32)
    K[:, 0] = 127.0
    q = rng.standard_normal((G, d)).astype(np.float32)
    kq, sc = oracle.quantize_rows(K)
    assert np.all(sc == 1.0)
    pool, _ = oracle.propose_row(q, kq, sc, 50)
    idx, _ = oracle.refine_row(q, K, np.arange(L, dtype=np.int32), 50)
    assert np.array_equal(pool, idx)


# ---------------------------------------------------------------- attention

@pytest.mark.parametrize("case", GOLD["attend"], ids=lambda c: c["cite"][:30])
def test_attend_hand_cases(case):
    out, lse = oracle.attend(np.array(case["q"], np.float32), np.array(case["K"], np.float32),
                             np.array(case["V"], np.float32), None, case["scale"])
    assert np.allclose(out, case["out"], rtol=1e-6, atol=1e-6)
    assert abs(lse - case["lse"]) < 1e-6


def test_dense_attend_matches_textbook_softmax():
    rng = np.random.default_rng(9)
    d, L = 64, 333
    q = rng.standard_normal(d).astype(np.float32)
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = rng.standard_normal((L, d)).astype(np.float32)
    sc = 1 / math.sqrt(d)
    out, lse = oracle.attend(q, K, V, None, sc)
    l = (K.astype(np.float64) @ q.astype(np.float64)) * sc
    w = np.exp(l - l.max())
    w /= w.sum()
    assert np.allclose(out, w @ V.astype(np.float64), rtol=0, atol=1e-6)
    assert abs(lse - (l.max() + math.log(np.exp(l - l.max()).sum()))) < 1e-5
    # sparse attention over every position is dense attention
    out2, lse2 = oracle.attend(q, K, V, np.arange(L, dtype=np.int32), sc)
    assert np.array_equal(out, out2) and lse == lse2
    # a subset attends only to its rows: reordering the rows does not matter
    sel = np.sort(rng.choice(L, 40, replace=False)).astype(np.int32)
    out3, _ = oracle.attend(q, K, V, sel, sc)
    out4, _ = oracle.attend(q, K[sel], V[sel], None, sc)
    assert np.allclose(out3, out4, atol=1e-7)


def test_attend_special_cases():
    rng = np.random.default_rng(10)
    d, L = 32, 50
    q = rng.standard_normal(d).astype(np.float32)
    V = rng.standard_normal((L, d)).astype(np.float32)
    # all keys equal -> uniform weights -> mean of V
    K = np.tile(rng.standard_normal(d).astype(np.float32), (L, 1))
    out, lse = oracle.attend(q, K, V, None, 0.3)
    assert np.allclose(out, V.astype(np.float64).mean(0), atol=1e-6)
    # weights sum to one: V of ones gives ones
    K = rng.standard_normal((L, d)).astype(np.float32) * 4
    out, _ = oracle.attend(q, K, np.ones((L, d), np.float32), None, 0.5)
    assert np.allclose(out, 1.0, atol=1e-6)
    # empty set
    out, lse = oracle.attend(q, K, V, np.zeros(0, np.int32), 0.5)
    assert np.all(out == 0) and lse == -math.inf


# ---------------------------------------------------------------- pipeline

def test_pipeline_tiny_invariants_and_recall():
    from kv_cache_top_proposal_b200 import workload

    cfg = workload.config("tiny")
    layers = list(workload.generate(cfg, "cpu"))
    res = pipeline.decode_step(cfg, layers)
    sal = workload.salient_positions(cfg)
    for r in res:
        pc, c = int(r["pool_cnt"][0, 0]), int(r["cnt"][0, 0])
        pool, idx = r["pool"][0, 0, :pc], r["idx"][0, 0, :c]
        assert pc == cfg.kappa_p and c == cfg.kappa
        assert np.all(np.diff(pool) > 0) and np.all(np.diff(idx) > 0)
        assert set(idx.tolist()) <= set(pool.tolist())
        assert np.all(r["pool"][0, 0, pc:] == -1) and np.all(r["idx"][0, 0, c:] == -1)
        # sanity (not parity): the planted salient positions are recalled
        hit = np.isin(sal[0][0].numpy(), idx).mean()
        assert hit >= 0.9, hit
        assert np.all(np.isfinite(r["out"]))


def test_pipeline_full_budget_equals_dense():
    from kv_cache_top_proposal_b200 import workload

    cfg = workload.config("tiny").replace(seqlens=(200,), kappa_p=200, kappa=200, num_layers=2)
    layers = list(workload.generate(cfg, "cpu"))
    res = pipeline.decode_step(cfg, layers)
    for lay, r in zip(layers, res):
        assert np.array_equal(r["idx"][0, 0], np.arange(200))
        dout, dlse = pipeline.attend_layer(lay.q, lay.k, lay.v, cfg.cu_seqlens, None, None)
        assert np.allclose(r["out"], dout, atol=1e-6)
        assert np.allclose(r["lse"], dlse, atol=1e-5)

"""CUDA path vs the CPU oracle, stage by stage, on identical inputs.

Every stage gets the same inputs on both sides (the GPU's own upstream index
set is handed to the oracle for the downstream stage, so a permitted
near-tie swap upstream cannot cascade).  Quantized keys and scales must be
bit-exact; index sets may differ only by near-ties (parity_util); attention
outputs must agree within 2e-3 max-abs for bf16 caches and 1e-5 for fp32.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import pipeline
from parity_util import atol_for, check_index_set

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def P(prism_lib):
    return prism_lib


def _np(t):
    return t.detach().float().cpu().numpy() if t.dtype not in (torch.int32, torch.int8, torch.int64) \
        else t.detach().cpu().numpy()


def make_case(seqlens, hq, hkv, d, dtype, seed=0, scale_rows=False):
    g = torch.Generator(device="cpu").manual_seed(seed)
    T = int(sum(seqlens))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = torch.randn((len(seqlens), hq, d), generator=g)
    k = torch.randn((hkv, T, d), generator=g)
    v = torch.randn((hkv, T, d), generator=g)
    if scale_rows:
        k = k * torch.exp(torch.randn((hkv, T, 1), generator=g) * 3)
    return q.to(tdt).to(DEV), k.to(tdt).to(DEV), v.to(tdt).to(DEV)


def problem(P, seqlens, hq, hkv, d, dtype):
    return P.Problem(seqlens, hq, hkv, d, P.BF16 if dtype == "bf16" else P.F32, device=DEV)


def ws_for(P, prob, op, kp=0, k=0):
    w = torch.zeros(P.workspace_size(prob, op, kp, k), dtype=torch.uint8, device=DEV)
    return w


# ------------------------------------------------------------------ quantize

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
def test_quantize_bit_exact(P, dtype, d):
    seqlens = [1000, 37, 0, 2049]
    prob = problem(P, seqlens, 8, 4, d, dtype)
    _, k, _ = make_case(seqlens, 8, 4, d, dtype, seed=1, scale_rows=True)
    k[0, 5] = 0  # an all-zero row
    k[1, 7, :] = 0
    k[1, 7, 3] = -2.5e-3
    T = prob.total_tokens
    kq = torch.zeros((4, T, d), dtype=torch.int8, device=DEV)
    sc = torch.zeros((4, T), dtype=torch.float32, device=DEV)
    ws = ws_for(P, prob, P.OP_QUANTIZE)
    P.quantize_k(prob, k, kq, sc, ws=ws)
    okq, osc = oracle.quantize_rows(_np(k).reshape(-1, d))
    assert np.array_equal(_np(kq).reshape(-1, d), okq)
    assert np.array_equal(_np(sc).reshape(-1).view(np.uint32), osc.view(np.uint32))
    # token-row path: only the listed rows change
    rows = torch.tensor([0, 999, 1037, T - 1], dtype=torch.int32, device=DEV)
    kq2 = torch.full_like(kq, 55)
    sc2 = torch.full_like(sc, -1.0)
    P.quantize_k(prob, k, kq2, sc2, tok_rows=rows, ws=ws)
    r = rows.cpu().numpy()
    assert np.array_equal(_np(kq2)[:, r], _np(kq)[:, r])
    assert np.array_equal(_np(sc2)[:, r], _np(sc)[:, r])
    mask = np.ones(T, bool)
    mask[r] = False
    assert np.all(_np(kq2)[:, mask] == 55) and np.all(_np(sc2)[:, mask] == -1.0)
    assert P.get_device_status(ws) == 0


# ------------------------------------------------------------------ propose

PROPOSE_CASES = [
    # seqlens, hq, hkv, d, dtype, kappa_p
    ([1024], 4, 1, 64, "f32", 256),
    ([5000, 1031, 0, 300], 8, 2, 128, "bf16", 1024),
    ([3000, 777], 8, 8, 64, "bf16", 200),       # G = 1
    ([2500], 64, 8, 128, "bf16", 333),          # G = 8
    ([1800], 32, 2, 64, "bf16", 500),           # G = 16
    ([1024, 1025, 1023], 16, 4, 128, "bf16", 1024),  # L == kappa_p, +-1
    ([40000], 8, 2, 128, "bf16", 4096),         # many tiles and chunks
    ([9000], 12, 3, 128, "f32", 700),           # G = 4, fp32
    ([1500, 77], 4, 4, 128, "bf16", 300),       # G = 1 at d = 128 (one head of the quad)
    ([2049, 100], 6, 2, 128, "bf16", 512),      # G = 3
    ([1700], 12, 2, 128, "bf16", 400),          # G = 6 (two quads, the second partial)
]


@pytest.mark.parametrize("case", PROPOSE_CASES, ids=lambda c: f"{c[0]}-{c[1]}/{c[2]}-d{c[3]}-{c[4]}-kp{c[5]}")
@pytest.mark.parametrize("scorer", ["i8", "tma", "mma", "simt"])
def test_propose_vs_oracle(P, case, scorer, monkeypatch):
    """i8: the default scorer, integer tensor cores on the stored codes with
    the query in fixed point, fed by tensor copies (d = 128 and G <= 8; d = 64
    takes the cp.async fp16 one, G > 8 the tensor-copy fp16 one); tma: the
    tensor-copy fp16 scorer; mma: the cp.async fp16 scorer; simt: CUDA cores."""
    seqlens, hq, hkv, d, dtype, kp = case
    if scorer == "simt":
        monkeypatch.setenv("PRISM_PROPOSE_SCORER", "simt")
    elif dtype != "bf16":
        pytest.skip("the tensor-core scorers take bf16 queries")
    elif scorer in ("mma", "tma"):
        monkeypatch.setenv("PRISM_PROPOSE_SCORER", scorer)
    prob = problem(P, seqlens, hq, hkv, d, dtype)
    q, k, _ = make_case(seqlens, hq, hkv, d, dtype, seed=2)
    T = prob.total_tokens
    kq = torch.zeros((hkv, T, d), dtype=torch.int8, device=DEV)
    sc = torch.zeros((hkv, T), dtype=torch.float32, device=DEV)
    P.quantize_k(prob, k, kq, sc)
    pool = torch.full((len(seqlens), hkv, kp), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((len(seqlens), hkv), -7, dtype=torch.int32, device=DEV)
    ws = ws_for(P, prob, P.OP_PROPOSE, kp)
    P.propose(prob, q, kq, sc, kp, pool, cnt, ws)
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    gscores = _np(ws[256:256 + hkv * T * 4].view(torch.float32)).reshape(hkv, T)
    opool, ocnt, oscores = pipeline.propose_layer(q, kq, sc, prob.cu_host.tolist(), kp)
    gp, gc = _np(pool), _np(cnt)
    assert np.array_equal(gc, ocnt)
    cu = prob.cu_host
    for b in range(len(seqlens)):
        for h in range(hkv):
            s = oscores[(b, h)]
            n = int(ocnt[b, h])
            if n:
                gs = gscores[h, cu[b]:cu[b + 1]]
                assert np.allclose(gs, s, rtol=2e-6, atol=2e-6 * np.abs(s).max()), (b, h)
            check_index_set(gp[b, h, :n], opool[b, h, :n], lambda t: s[t], f"pool b{b} h{h}")
            assert np.all(gp[b, h, n:] == -1)


@pytest.mark.parametrize("keys", ["int8", "int2"])
def test_propose_workspace_reuse(P, keys):
    """Calls on one propose workspace (here three, on different queries) each
    match the oracle: nothing a call leaves in the workspace (scores,
    first-digit histograms) leaks into the next."""
    seqlens, hq, hkv, d, kp = [5000, 2100], 8, 2, 128, 900
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    T = prob.total_tokens
    ws = ws_for(P, prob, P.OP_PROPOSE, kp)
    for it in range(3):
        q, k, _ = make_case(seqlens, hq, hkv, d, "bf16", seed=40 + it)
        pool = torch.full((len(seqlens), hkv, kp), -7, dtype=torch.int32, device=DEV)
        cnt = torch.full((len(seqlens), hkv), -7, dtype=torch.int32, device=DEV)
        if keys == "int8":
            kq = torch.zeros((hkv, T, d), dtype=torch.int8, device=DEV)
            sc = torch.zeros((hkv, T), dtype=torch.float32, device=DEV)
            P.quantize_k(prob, k, kq, sc)
            P.propose(prob, q, kq, sc, kp, pool, cnt, ws)
            opool, ocnt, oscores = pipeline.propose_layer(q, kq, sc, prob.cu_host.tolist(), kp)
        else:
            codes = torch.zeros((hkv, T, d // 4), dtype=torch.uint8, device=DEV)
            params = torch.zeros((hkv, T, d // 32, 2), dtype=torch.int16, device=DEV)
            P.quantize_k_int2(prob, k, codes, params)
            P.propose_int2(prob, q, codes, params, kp, pool, cnt, ws)
            opool, ocnt, oscores = pipeline.propose_layer_int2(
                q, codes.cpu().numpy(), params.cpu().numpy().view(np.uint16), prob.cu_host.tolist(), kp)
        torch.cuda.synchronize()
        assert P.get_device_status(ws) == 0
        gp, gc = _np(pool), _np(cnt)
        assert np.array_equal(gc, ocnt)
        for b in range(len(seqlens)):
            for h in range(hkv):
                n = int(ocnt[b, h])
                sc_of = oscores[(b, h)]
                check_index_set(gp[b, h, :n], opool[b, h, :n], lambda t: sc_of[t], f"call {it} b{b} h{h}")


PROPOSE_APPEND_CASES = [
    # seqlens, hq, hkv, kappa_p
    ([5000, 1031, 0, 300, 1], 8, 2, 1024),  # ragged, an empty sequence, one of length 1
    ([2500, 129, 128], 64, 8, 333),          # G = 8; the new row alone in a stage, and at its end
    ([3000, 777], 8, 8, 200),                # G = 1
]


@pytest.mark.parametrize("agg", ["max", "sum"])
@pytest.mark.parametrize("case", PROPOSE_APPEND_CASES, ids=lambda c: f"{c[0]}-{c[1]}/{c[2]}-kp{c[3]}")
def test_propose_append_vs_oracle(P, case, agg):
    """prism_propose_append: the scorer quantizes this token's key rows into
    kq / k_scale at L_b - 1 (bit-exact with the oracle's quantizer; every
    other row untouched) and scores them with the rest; the pool matches the
    oracle's proposal over the codes with the new rows in place.  The cache
    row at L_b - 1 holds something else (the new row is appended later)."""
    seqlens, hq, hkv, kp = case
    d = 128
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    q, k, _ = make_case(seqlens, hq, hkv, d, "bf16", seed=31)
    g = torch.Generator(device="cpu").manual_seed(32)
    k_new = (torch.randn((len(seqlens), hkv, d), generator=g) * 1.5).to(torch.bfloat16).to(DEV)
    k_new[0, 0, :] = 0  # an all-zero new row: scale 0, codes 0
    T = prob.total_tokens
    kq = torch.zeros((hkv, T, d), dtype=torch.int8, device=DEV)
    sc = torch.zeros((hkv, T), dtype=torch.float32, device=DEV)
    P.quantize_k(prob, k, kq, sc)  # the cache's codes, stale at L_b - 1
    kq_before, sc_before = _np(kq).copy(), _np(sc).copy()
    pool = torch.full((len(seqlens), hkv, kp), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((len(seqlens), hkv), -7, dtype=torch.int32, device=DEV)
    ws = ws_for(P, prob, P.OP_PROPOSE, kp)
    P.propose_append(prob, q, k_new, kq, sc, kp, pool, cnt, ws, sum_group=agg == "sum")
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    cu = prob.cu_host
    want_kq, want_sc = kq_before.copy(), sc_before.copy()
    okq, osc = oracle.quantize_rows(_np(k_new).reshape(-1, d))
    okq, osc = okq.reshape(len(seqlens), hkv, d), osc.reshape(len(seqlens), hkv)
    for b in range(len(seqlens)):
        if cu[b + 1] > cu[b]:
            want_kq[:, cu[b + 1] - 1] = okq[b]
            want_sc[:, cu[b + 1] - 1] = osc[b]
    assert np.array_equal(_np(kq), want_kq)
    assert np.array_equal(_np(sc).view(np.uint32), want_sc.view(np.uint32))
    opool, ocnt, oscores = pipeline.propose_layer(q, want_kq, want_sc, cu.tolist(), kp, agg=agg)
    gp, gc = _np(pool), _np(cnt)
    assert np.array_equal(gc, ocnt)
    gscores = _np(ws[256:256 + hkv * T * 4].view(torch.float32)).reshape(hkv, T)
    for b in range(len(seqlens)):
        for h in range(hkv):
            n = int(ocnt[b, h])
            s_ = oscores[(b, h)]
            if n:
                gs = gscores[h, cu[b]:cu[b + 1]]
                assert np.allclose(gs, s_, rtol=2e-6, atol=2e-6 * np.abs(s_).max()), (b, h)
            check_index_set(gp[b, h, :n], opool[b, h, :n], lambda t: s_[t], f"pool b{b} h{h}")
            assert np.all(gp[b, h, n:] == -1)


def test_propose_append_unsupported(P):
    """Shapes the integer scorer does not take are refused, not computed."""
    prob = problem(P, [300], 8, 2, 64, "bf16")  # d = 64
    q, k, _ = make_case([300], 8, 2, 64, "bf16", seed=3)
    kq = torch.zeros((2, 300, 64), dtype=torch.int8, device=DEV)
    sc = torch.zeros((2, 300), dtype=torch.float32, device=DEV)
    pool = torch.zeros((1, 2, 100), dtype=torch.int32, device=DEV)
    cnt = torch.zeros((1, 2), dtype=torch.int32, device=DEV)
    k_new = torch.zeros((1, 2, 64), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(P.PrismError) as e:
        P.propose_append(prob, q, k_new, kq, sc, 100, pool, cnt, ws_for(P, prob, P.OP_PROPOSE, 100))
    assert e.value.status == P.ERR_UNSUPPORTED


def test_propose_query_ranges(P):
    """Query heads far from unit scale, where the integer scorer's fixed-point
    query needs care: a group at 2^-110 (shift above 126, taken in two
    factors), one at 2^100, one whose heads mix elements 2^-40 apart (the
    small ones off the grid), and one with an all-zero head and an all-negative
    one.  Scores and pools are checked against the oracle as above."""
    seqlens, hq, hkv, d, kp = [3000, 1200], 16, 4, 128, 700
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    q, k, _ = make_case(seqlens, hq, hkv, d, "bf16", seed=11)
    qf = q.float().cpu().view(len(seqlens), hkv, hq // hkv, d)
    qf[:, 0] *= 2.0 ** -110
    qf[:, 1] *= 2.0 ** 100
    qf[:, 2, :, ::2] *= 2.0 ** -40
    qf[:, 3, 0] = 0.0
    qf[:, 3, 1] = -qf[:, 3, 1].abs()
    q = qf.view(len(seqlens), hq, d).to(torch.bfloat16).to(DEV)
    T = prob.total_tokens
    kq = torch.zeros((hkv, T, d), dtype=torch.int8, device=DEV)
    sc = torch.zeros((hkv, T), dtype=torch.float32, device=DEV)
    P.quantize_k(prob, k, kq, sc)
    pool = torch.full((len(seqlens), hkv, kp), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((len(seqlens), hkv), -7, dtype=torch.int32, device=DEV)
    ws = ws_for(P, prob, P.OP_PROPOSE, kp)
    P.propose(prob, q, kq, sc, kp, pool, cnt, ws)
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    gscores = _np(ws[256:256 + hkv * T * 4].view(torch.float32)).reshape(hkv, T)
    opool, ocnt, oscores = pipeline.propose_layer(q, kq, sc, prob.cu_host.tolist(), kp)
    gp, gc = _np(pool), _np(cnt)
    assert np.array_equal(gc, ocnt)
    cu = prob.cu_host
    for b in range(len(seqlens)):
        for h in range(hkv):
            s = oscores[(b, h)]
            n = int(ocnt[b, h])
            gs = gscores[h, cu[b]:cu[b + 1]]
            assert np.all(np.isfinite(gs)) and np.abs(s).max() > 0, (b, h)
            assert np.allclose(gs, s, rtol=2e-6, atol=2e-6 * np.abs(s).max()), (b, h)
            check_index_set(gp[b, h, :n], opool[b, h, :n], lambda t: s[t], f"pool b{b} h{h}")


@pytest.mark.parametrize("seqlens,cap,kp", [
    ([32768, 300], None, 4096),     # 4-CTA clusters, the long row filling all four
    ([32769, 300], None, 4096),     # one position more: 8-CTA clusters
    ([65536, 10], None, 8192),      # 8-CTA clusters, full
    ([1000, 2000], 43000, 700),     # short rows, but the last may grow to 42000: 8
    ([70000, 4000], None, 6000),    # 16-CTA clusters
], ids=["cl4-full", "cl8-edge", "cl8-full", "cl8-by-capacity", "cl16"])
def test_propose_select_cluster_sizes(P, seqlens, cap, kp):
    """The proposal selection's cluster is the smallest (4, 8 or 16 CTAs of
    8192 keys) that holds the longest row the call can meet, the last row
    counted up to the capacity.  Pools match the oracle's on each side of
    the boundaries; the spare rows past the end hold valid codes that must
    stay out of the last row's pool."""
    hq, hkv, d = 8, 2, 128
    prob = P.Problem(seqlens, hq, hkv, d, P.BF16, device=DEV, capacity=cap)
    T = prob.total_tokens
    q, k, _ = make_case(list(seqlens) + ([T - sum(seqlens)] if cap else []), hq, hkv, d,
                        "bf16", seed=21)
    kq = torch.zeros((hkv, T, d), dtype=torch.int8, device=DEV)
    sc = torch.zeros((hkv, T), dtype=torch.float32, device=DEV)
    P.quantize_k(P.Problem([T], hq, hkv, d, P.BF16, device=DEV), k, kq, sc)
    q = q[:len(seqlens)].contiguous()
    pool = torch.full((len(seqlens), hkv, kp), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((len(seqlens), hkv), -7, dtype=torch.int32, device=DEV)
    ws = ws_for(P, prob, P.OP_PROPOSE, kp)
    P.propose(prob, q, kq, sc, kp, pool, cnt, ws)
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    opool, ocnt, oscores = pipeline.propose_layer(q, kq, sc, prob.cu_host.tolist(), kp)
    gp, gc = _np(pool), _np(cnt)
    assert np.array_equal(gc, ocnt)
    for b in range(len(seqlens)):
        for h in range(hkv):
            s = oscores[(b, h)]
            n = int(ocnt[b, h])
            check_index_set(gp[b, h, :n], opool[b, h, :n], lambda t: s[t], f"pool b{b} h{h}")
            assert np.all(gp[b, h, n:] == -1)


@pytest.mark.parametrize("L0,kp", [(3000, 1000), (60000, 8192)], ids=["small", "many-candidates"])
def test_propose_all_ties_lower_index_wins(P, L0, kp):
    """Equal scores: the lowest positions win.  At 60000 positions every CTA of
    the selection holds more first-digit candidates than rank 0 ranks, so the
    cluster-wide digit rounds run."""
    seqlens, hq, hkv, d = [L0, 500], 8, 2, 128
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    q, k, _ = make_case(seqlens, hq, hkv, d, "bf16", seed=3)
    k[:] = k[:, :1]  # every key row identical -> every score equal
    T = prob.total_tokens
    kq = torch.zeros((hkv, T, d), dtype=torch.int8, device=DEV)
    sc = torch.zeros((hkv, T), dtype=torch.float32, device=DEV)
    P.quantize_k(prob, k, kq, sc)
    pool = torch.zeros((2, hkv, kp), dtype=torch.int32, device=DEV)
    cnt = torch.zeros((2, hkv), dtype=torch.int32, device=DEV)
    P.propose(prob, q, kq, sc, kp, pool, cnt, ws_for(P, prob, P.OP_PROPOSE, kp))
    gp = _np(pool)
    for h in range(hkv):
        assert np.array_equal(gp[0, h], np.arange(kp))
        assert np.array_equal(gp[1, h, :500], np.arange(500)) and np.all(gp[1, h, 500:] == -1)
    assert _np(cnt).tolist() == [[kp, kp], [500, 500]]


# ------------------------------------------------------------------ refine

REFINE_CASES = [
    ([1024], 4, 1, 64, "f32", 256, 64),
    ([5000, 1031, 0, 300], 8, 2, 128, "bf16", 1024, 256),
    ([3000, 777], 8, 8, 64, "bf16", 200, 200),   # rho = 1: idx == pool
    ([2500], 64, 8, 128, "bf16", 333, 100),
    ([1800], 32, 2, 64, "bf16", 500, 17),
    ([40000], 8, 2, 128, "bf16", 8192, 2048),
]


@pytest.mark.parametrize("case", REFINE_CASES, ids=lambda c: f"{c[0]}-{c[1]}/{c[2]}-d{c[3]}-{c[4]}-{c[5]}-{c[6]}")
def test_refine_vs_oracle(P, case):
    seqlens, hq, hkv, d, dtype, kp, kap = case
    B = len(seqlens)
    prob = problem(P, seqlens, hq, hkv, d, dtype)
    q, k, _ = make_case(seqlens, hq, hkv, d, dtype, seed=4)
    cu = prob.cu_host
    # an arbitrary ascending pool per row (what a proposal layer hands over)
    rng = np.random.default_rng(5)
    pool = np.full((B, hkv, kp), -1, np.int32)
    pcnt = np.zeros((B, hkv), np.int32)
    for b, L in enumerate(seqlens):
        for h in range(hkv):
            n = min(kp, L)
            pool[b, h, :n] = np.sort(rng.choice(L, n, replace=False))
            pcnt[b, h] = n
    dpool = torch.tensor(pool, device=DEV)
    dcnt = torch.tensor(pcnt, device=DEV)
    idx = torch.full((B, hkv, kap), -7, dtype=torch.int32, device=DEV)
    cnt = torch.zeros((B, hkv), dtype=torch.int32, device=DEV)
    logits = torch.full((B, hq, kap), 12345.0, device=DEV)
    ws = ws_for(P, prob, P.OP_REFINE, kp, kap)
    P.refine(prob, q, k, dpool, dcnt, kp, kap, idx, cnt, ws, logits=logits)
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    oidx, ocnt, oscores = pipeline.refine_layer(q, k, cu.tolist(), pool, pcnt, kap)
    gi, gc, gl = _np(idx), _np(cnt), _np(logits)
    assert np.array_equal(gc, ocnt)
    qn, kn = _np(q).astype(np.float64), _np(k).astype(np.float64)
    G = hq // hkv
    for b in range(B):
        for h in range(hkv):
            n = int(pcnt[b, h])
            r = dict(zip(pool[b, h, :n].tolist(), oscores[(b, h)].tolist()))
            c = int(ocnt[b, h])
            check_index_set(gi[b, h, :c], oidx[b, h, :c], lambda t: r[t], f"idx b{b} h{h}")
            assert set(gi[b, h, :c].tolist()) <= set(pool[b, h, :n].tolist())
            assert np.all(gi[b, h, c:] == -1)
            if c:
                rows = kn[h, cu[b] + gi[b, h, :c]]
                want = qn[b, h * G:(h + 1) * G] @ rows.T
                got = gl[b, h * G:(h + 1) * G, :c]
                assert np.allclose(got, want, rtol=1e-5, atol=1e-4), (b, h)
            assert np.all(gl[b, h * G:(h + 1) * G, c:] == 12345.0)


# ------------------------------------------------------------------ attention

MASS_CASES = [
    # (seqlens, Hq, Hkv, d, dtype, kappa_p, kappa): one head (mass order is
    # score order), groups of 4 / 8 / 16, d = 64, fp32, a ragged batch with
    # an empty sequence, pools of 8192, kappa = kappa_p
    ([5000], 4, 4, 128, "bf16", 1024, 256),
    ([20000, 3000, 0, 777], 32, 8, 128, "bf16", 4096, 1024),
    ([30000], 16, 2, 128, "bf16", 8192, 2048),
    ([9000], 16, 1, 64, "bf16", 2048, 300),
    ([4000, 1500], 8, 2, 64, "f32", 1000, 1000),
]


@pytest.mark.parametrize("case", MASS_CASES, ids=lambda c: f"{len(c[0])}seq-{c[1]}/{c[2]}-d{c[3]}-{c[4]}-kp{c[5]}-k{c[6]}")
def test_refine_mass_vs_oracle(P, case):
    """prism_refine_mass against the oracle's softmax-mass selection, every
    row: counts exact, sets up to near-ties of the fp64 mass, -1 padding."""
    seqlens, hq, hkv, d, dtype, kp, kap = case
    B = len(seqlens)
    prob = problem(P, seqlens, hq, hkv, d, dtype)
    q, k, v = make_case(seqlens, hq, hkv, d, dtype, seed=41)
    rng = np.random.default_rng(42)
    pool = np.full((B, hkv, kp), -1, np.int32)
    pcnt = np.zeros((B, hkv), np.int32)
    for b, L in enumerate(seqlens):
        for h in range(hkv):
            n = min(kp, L)
            pool[b, h, :n] = np.sort(rng.choice(L, n, replace=False))
            pcnt[b, h] = n
    scale = float(np.float32(1 / math.sqrt(d)))
    ws = ws_for(P, prob, P.OP_REFINE, kp, kap)
    idx = torch.full((B, hkv, kap), -7, dtype=torch.int32, device=DEV)
    cnt = torch.zeros((B, hkv), dtype=torch.int32, device=DEV)
    P.refine_mass(prob, q, k, torch.tensor(pool, device=DEV), torch.tensor(pcnt, device=DEV), kp, kap,
                  scale, idx, cnt, ws)
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    oidx, ocnt, omass = pipeline.refine_layer(q, k, prob.cu_host.tolist(), pool, pcnt, kap, agg="mass",
                                              softmax_scale=scale)
    gi, gc = _np(idx), _np(cnt)
    assert np.array_equal(gc, ocnt)
    for b in range(B):
        for h in range(hkv):
            n, c = int(pcnt[b, h]), int(ocnt[b, h])
            r = dict(zip(pool[b, h, :n].tolist(), omass[(b, h)].tolist()))
            check_index_set(gi[b, h, :c], oidx[b, h, :c], lambda t: r[t], f"mass b{b} h{h}")
            assert np.all(gi[b, h, c:] == -1)


ATTEND_CASES = [
    ([1024], 4, 1, 64, "f32", 64),
    ([5000, 1031, 0, 300], 8, 2, 128, "bf16", 256),
    ([3000, 777], 8, 8, 64, "bf16", 200),
    ([2500], 64, 8, 128, "bf16", 100),
    ([1800], 32, 2, 64, "bf16", 17),
    ([40000], 8, 2, 128, "bf16", 2048),
    ([700, 2], 16, 1, 128, "f32", 1000),
]


@pytest.mark.parametrize("case", ATTEND_CASES, ids=lambda c: f"{c[0]}-{c[1]}/{c[2]}-d{c[3]}-{c[4]}-{c[5]}")
def test_sparse_decode_vs_oracle(P, case):
    seqlens, hq, hkv, d, dtype, kap = case
    B = len(seqlens)
    prob = problem(P, seqlens, hq, hkv, d, dtype)
    q, k, v = make_case(seqlens, hq, hkv, d, dtype, seed=6)
    rng = np.random.default_rng(7)
    idx = np.full((B, hkv, kap), -1, np.int32)
    cnt = np.zeros((B, hkv), np.int32)
    for b, L in enumerate(seqlens):
        for h in range(hkv):
            n = min(kap, L) if (b + h) % 3 else min(kap, L) // 2
            idx[b, h, :n] = np.sort(rng.choice(L, n, replace=False))
            cnt[b, h] = n
    out = torch.full((B, hq, d), 77.0, device=DEV)
    lse = torch.full((B, hq), 77.0, device=DEV)
    ws = ws_for(P, prob, P.OP_SPARSE_DECODE, 0, kap)
    scale = float(np.float32(1 / math.sqrt(d)))
    P.sparse_decode(prob, q, k, v, torch.tensor(idx, device=DEV), torch.tensor(cnt, device=DEV),
                    kap, scale, out, ws, lse=lse)
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    oout, olse = pipeline.attend_layer(q, k, v, prob.cu_host.tolist(), idx, cnt, scale)
    tol = atol_for(dtype)
    assert np.abs(_np(out) - oout).max() <= tol
    gl = _np(lse)
    fin = np.isfinite(olse)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.abs(gl[fin] - olse[fin]).max() <= tol * 10
    assert np.all(_np(out)[~fin] == 0)


@pytest.mark.parametrize("case", [([1024], 4, 1, 64, "f32"), ([5000, 1031, 0, 300], 8, 2, 128, "bf16"),
                                  ([20000], 32, 8, 128, "bf16"), ([999], 16, 1, 64, "bf16"),
                                  ([70000, 3, 129, 12345], 16, 2, 128, "bf16"),
                                  ([4097, 1], 8, 8, 64, "bf16"), ([3000, 200], 6, 3, 128, "bf16"),
                                  ([2000], 32, 2, 128, "bf16")],
                         ids=lambda c: f"{c[0]}-{c[1]}/{c[2]}-d{c[3]}-{c[4]}")
def test_dense_decode_vs_oracle(P, case):
    seqlens, hq, hkv, d, dtype = case
    prob = problem(P, seqlens, hq, hkv, d, dtype)
    q, k, v = make_case(seqlens, hq, hkv, d, dtype, seed=8)
    out = torch.zeros((len(seqlens), hq, d), device=DEV)
    lse = torch.zeros((len(seqlens), hq), device=DEV)
    scale = float(np.float32(1 / math.sqrt(d)))
    ws = ws_for(P, prob, P.OP_DENSE_DECODE)
    P.dense_decode(prob, q, k, v, scale, out, ws, lse=lse)
    torch.cuda.synchronize()
    oout, olse = pipeline.attend_layer(q, k, v, prob.cu_host.tolist(), None, None, scale)
    tol = atol_for(dtype)
    assert np.abs(_np(out) - oout).max() <= tol
    fin = np.isfinite(olse)
    assert np.abs(_np(lse)[fin] - olse[fin]).max() <= tol * 10


def test_dense_decode_ignores_rows_past_the_end(P):
    """Cache rows past a sequence's end (the next sequence's, and spare rows
    holding NaN) share the dense pass's 128-row stages with the last valid
    rows: they carry no weight and their bytes never reach the output."""
    seqlens, hq, hkv, d = [1000, 777], 8, 2, 128
    cap = 2000
    prob = P.Problem(seqlens, hq, hkv, d, P.BF16, device=DEV, capacity=cap)
    q, k0, v0 = make_case(seqlens, hq, hkv, d, "bf16", seed=12)
    k = torch.full((hkv, cap, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    v = torch.full((hkv, cap, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    k[:, :1777], v[:, :1777] = k0, v0
    out = torch.zeros((2, hq, d), device=DEV)
    lse = torch.zeros((2, hq), device=DEV)
    scale = float(np.float32(1 / math.sqrt(d)))
    ws = ws_for(P, prob, P.OP_DENSE_DECODE)
    P.dense_decode(prob, q, k, v, scale, out, ws, lse=lse)
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    oout, olse = pipeline.attend_layer(q, k0, v0, [0, 1000, 1777], None, None, scale)
    assert np.all(np.isfinite(_np(out)))
    assert np.abs(_np(out) - oout).max() <= atol_for("bf16")
    assert np.abs(_np(lse) - olse).max() <= atol_for("bf16") * 10


def test_full_budget_sparse_equals_dense(P):
    seqlens, hq, hkv, d = [600, 257], 8, 2, 128
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    q, k, v = make_case(seqlens, hq, hkv, d, "bf16", seed=9)
    kap = 600
    idx = torch.full((2, hkv, kap), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros((2, hkv), dtype=torch.int32, device=DEV)
    for b, L in enumerate(seqlens):
        idx[b, :, :L] = torch.arange(L, device=DEV, dtype=torch.int32)
        cnt[b] = L
    scale = 0.1
    o1 = torch.zeros((2, hq, d), device=DEV)
    o2 = torch.zeros((2, hq, d), device=DEV)
    P.sparse_decode(prob, q, k, v, idx, cnt, kap, scale, o1, ws_for(P, prob, P.OP_SPARSE_DECODE, 0, kap))
    P.dense_decode(prob, q, k, v, scale, o2, ws_for(P, prob, P.OP_DENSE_DECODE))
    assert (o1 - o2).abs().max().item() <= 1e-5


def test_bad_indices_flagged_not_read(P):
    seqlens, hq, hkv, d, kap = [300], 4, 1, 128, 8
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    q, k, v = make_case(seqlens, hq, hkv, d, "bf16", seed=10)
    idx = torch.tensor([[[0, 5, 299, 300, -3, 1 << 30, 7, 8]]], dtype=torch.int32, device=DEV)
    cnt = torch.tensor([[8]], dtype=torch.int32, device=DEV)
    ws = ws_for(P, prob, P.OP_SPARSE_DECODE, 0, kap)
    out = torch.zeros((1, hq, d), device=DEV)
    P.sparse_decode(prob, q, k, v, idx, cnt, kap, 0.1, out, ws)
    assert P.get_device_status(ws) & P.DEV_BAD_INDEX
    good = np.array([0, 5, 299, 7, 8], np.int32)
    oout, _ = pipeline.attend_layer(q, k, v, [0, 300], good[None, None], np.array([[5]]), 0.1)
    assert np.abs(_np(out) - oout).max() <= 2e-3
    P.clear_device_status(ws)
    assert P.get_device_status(ws) == 0


# ------------------------------------------------------------------ fused refine + decode

@pytest.mark.parametrize("agg", ["max", "sum"])
@pytest.mark.parametrize("case", REFINE_CASES + [([8192], 32, 8, 128, "bf16", 8192, 2048),
                                                  ([70000, 3], 8, 2, 64, "bf16", 6000, 1500)],
                         ids=lambda c: f"{c[0]}-{c[1]}/{c[2]}-d{c[3]}-{c[4]}-{c[5]}-{c[6]}")
def test_refine_decode_vs_oracle(P, case, agg):
    """agg: how the group's query heads combine into the exact score (the
    maximum, or the group-sum variant, PRISM_RD_SUM_GROUP)."""
    seqlens, hq, hkv, d, dtype, kp, kap = case
    B = len(seqlens)
    prob = problem(P, seqlens, hq, hkv, d, dtype)
    q, k, v = make_case(seqlens, hq, hkv, d, dtype, seed=12)
    cu = prob.cu_host
    rng = np.random.default_rng(13)
    pool = np.full((B, hkv, kp), -1, np.int32)
    pcnt = np.zeros((B, hkv), np.int32)
    for b, L in enumerate(seqlens):
        for h in range(hkv):
            n = min(kp, L)
            pool[b, h, :n] = np.sort(rng.choice(L, n, replace=False))
            pcnt[b, h] = n
    idx = torch.full((B, hkv, kap), -7, dtype=torch.int32, device=DEV)
    cnt = torch.zeros((B, hkv), dtype=torch.int32, device=DEV)
    out = torch.full((B, hq, d), 77.0, device=DEV)
    lse = torch.full((B, hq), 77.0, device=DEV)
    ws = ws_for(P, prob, P.OP_REFINE_DECODE, kp, kap)
    assert ws.numel() == 256
    scale = float(np.float32(1 / math.sqrt(d)))
    P.refine_decode(prob, q, k, v, torch.tensor(pool, device=DEV), torch.tensor(pcnt, device=DEV),
                    kp, kap, scale, idx, cnt, out, ws, lse=lse, sum_group=agg == "sum")
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    oidx, ocnt, oscores = pipeline.refine_layer(q, k, cu.tolist(), pool, pcnt, kap, agg=agg)
    gi, gc = _np(idx), _np(cnt)
    assert np.array_equal(gc, ocnt)
    for b in range(B):
        for h in range(hkv):
            n = int(pcnt[b, h])
            r = dict(zip(pool[b, h, :n].tolist(), oscores[(b, h)].tolist()))
            c = int(ocnt[b, h])
            check_index_set(gi[b, h, :c], oidx[b, h, :c], lambda t: r[t], f"idx b{b} h{h}")
            assert np.all(gi[b, h, c:] == -1)
    # attention over the GPU's own set (cascade control)
    oout, olse = pipeline.attend_layer(q, k, v, cu.tolist(), gi, gc, scale)
    tol = atol_for(dtype)
    assert np.abs(_np(out) - oout).max() <= tol
    gl = _np(lse)
    fin = np.isfinite(olse)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.abs(gl[fin] - olse[fin]).max() <= tol * 10
    assert np.all(_np(out)[~fin] == 0)


def test_refine_decode_ties_and_bad_positions(P):
    seqlens, hq, hkv, d, kp, kap = [4000], 8, 2, 128, 1000, 300
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    q, k, v = make_case(seqlens, hq, hkv, d, "bf16", seed=14)
    k[:, :] = k[:, :1]  # all scores equal: the lowest pool slots win
    pool = torch.arange(0, 4 * kp, 4, dtype=torch.int32, device=DEV).repeat(1, hkv, 1)
    cnt_p = torch.full((1, hkv), kp, dtype=torch.int32, device=DEV)
    idx = torch.zeros((1, hkv, kap), dtype=torch.int32, device=DEV)
    cnt = torch.zeros((1, hkv), dtype=torch.int32, device=DEV)
    out = torch.zeros((1, hq, d), device=DEV)
    ws = ws_for(P, prob, P.OP_REFINE_DECODE, kp, kap)
    P.refine_decode(prob, q, k, v, pool, cnt_p, kp, kap, 0.1, idx, cnt, out, ws)
    for h in range(hkv):
        assert np.array_equal(_np(idx)[0, h], np.arange(0, 4 * kap, 4))
    oout, _ = pipeline.attend_layer(q, k, v, [0, 4000], _np(idx), _np(cnt), 0.1)
    assert np.abs(_np(out) - oout).max() <= 2e-3
    assert P.get_device_status(ws) == 0
    # a pool position past the sequence is flagged, ranks last, carries no weight
    pool[0, 0, 5] = 4000
    P.refine_decode(prob, q, k, v, pool, cnt_p, kp, kap, 0.1, idx, cnt, out, ws)
    assert P.get_device_status(ws) & P.DEV_BAD_INDEX


def test_refine_decode_prefetch_changes_nothing(P):
    seqlens, hq, hkv, d, kp, kap = [20000], 8, 2, 128, 4096, 1024
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    q, k, v = make_case(seqlens, hq, hkv, d, "bf16", seed=15)
    k2 = torch.randn_like(k)
    rng = np.random.default_rng(16)
    pool = torch.tensor(np.sort(rng.choice(20000, (hkv, kp), replace=True), axis=1)[None], device=DEV)
    pool = torch.tensor(np.stack([np.sort(rng.choice(20000, kp, replace=False)) for _ in range(hkv)])[None],
                        dtype=torch.int32, device=DEV)
    cnt_p = torch.full((1, hkv), kp, dtype=torch.int32, device=DEV)
    ws = ws_for(P, prob, P.OP_REFINE_DECODE, kp, kap)
    res = []
    for kpf in (None, k2):
        idx = torch.zeros((1, hkv, kap), dtype=torch.int32, device=DEV)
        cnt = torch.zeros((1, hkv), dtype=torch.int32, device=DEV)
        out = torch.zeros((1, hq, d), device=DEV)
        P.refine_decode(prob, q, k, v, pool, cnt_p, kp, kap, 0.1, idx, cnt, out, ws, k_prefetch=kpf)
        res.append((idx, cnt, out))
    torch.cuda.synchronize()
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    assert torch.equal(res[0][2], res[1][2])
    assert P.get_device_status(ws) == 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_refine_decode_appends_new_rows(P, dtype):
    """Rows passed as k_new / v_new are written at position L_b - 1 and used
    there: the result equals prism_append_kv followed by the plain call, and
    the last position is in every pool (it must be read from the new rows)."""
    seqlens, hq, hkv, d, kp, kap = [5000, 2100, 1], 8, 2, 128, 1024, 256
    B = len(seqlens)
    prob = problem(P, seqlens, hq, hkv, d, dtype)
    q, k, v = make_case(seqlens, hq, hkv, d, dtype, seed=17)
    g = torch.Generator(device="cpu").manual_seed(18)
    k_new = (torch.randn((B, hkv, d), generator=g) * 3).to(k.dtype).to(DEV)
    v_new = torch.randn((B, hkv, d), generator=g).to(v.dtype).to(DEV)
    rng = np.random.default_rng(19)
    pool = np.full((B, hkv, kp), -1, np.int32)
    pcnt = np.zeros((B, hkv), np.int32)
    for b, L in enumerate(seqlens):
        for h in range(hkv):
            n = min(kp, L)
            sel = set(rng.choice(L, n, replace=False).tolist())
            if L - 1 not in sel:
                sel.discard(min(sel))
                sel.add(L - 1)
            pool[b, h, :n] = np.sort(np.array(sorted(sel)))
            pcnt[b, h] = n
    pool_t, pcnt_t = torch.tensor(pool, device=DEV), torch.tensor(pcnt, device=DEV)
    scale = float(np.float32(1 / math.sqrt(d)))
    ws = ws_for(P, prob, P.OP_REFINE_DECODE, kp, kap)
    res = []
    for fused in (False, True):
        kc, vc = k.clone(), v.clone()
        idx = torch.full((B, hkv, kap), -7, dtype=torch.int32, device=DEV)
        cnt = torch.zeros((B, hkv), dtype=torch.int32, device=DEV)
        out = torch.full((B, hq, d), 77.0, device=DEV)
        lse = torch.full((B, hq), 77.0, device=DEV)
        if fused:
            P.refine_decode(prob, q, kc, vc, pool_t, pcnt_t, kp, kap, scale, idx, cnt, out, ws,
                            lse=lse, k_new=k_new, v_new=v_new)
        else:
            P.append_kv(prob, k_new, v_new, kc, vc)
            P.refine_decode(prob, q, kc, vc, pool_t, pcnt_t, kp, kap, scale, idx, cnt, out, ws,
                            lse=lse)
        torch.cuda.synchronize()
        res.append((kc, vc, idx, cnt, out, lse))
    assert P.get_device_status(ws) == 0
    (k0, v0, i0, c0, o0, l0), (k1, v1, i1, c1, o1, l1) = res
    assert torch.equal(k0, k1) and torch.equal(v0, v1)
    assert torch.equal(i0, i1) and torch.equal(c0, c1)
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
    # the new rows took part: the last position is selected somewhere, and the
    # result matches the oracle on the appended cache
    gi, gc = _np(i1), _np(c1)
    assert any((gi[b, h, :gc[b, h]] == seqlens[b] - 1).any() for b in range(B) for h in range(hkv))
    # the index sets against the oracle's refine on the appended cache
    cu = prob.cu_host.tolist()
    oidx, ocnt, orr = pipeline.refine_layer(q, k1, cu, pool, pcnt, kap)
    for b in range(B):
        for h in range(hkv):
            n, c = int(pcnt[b, h]), int(ocnt[b, h])
            assert int(gc[b, h]) == c
            r = dict(zip(pool[b, h, :n].tolist(), orr[(b, h)].tolist()))
            check_index_set(gi[b, h, :c], oidx[b, h, :c], lambda t: r[t], f"append idx {b},{h}")
    oout, _ = pipeline.attend_layer(q, k1, v1, cu, gi, gc, scale)
    assert np.abs(_np(o1) - oout).max() <= atol_for(dtype)


def test_refine_decode_overlapped_launches_match(P):
    """Consecutive refined layers launched with PRISM_RD_OVERLAP (each may
    start before the previous one ends) give the results of plain launches."""
    seqlens, hq, hkv, d, kp, kap = [30000, 7000], 32, 8, 128, 4096, 1024
    B = len(seqlens)
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    rng = np.random.default_rng(21)
    pool = np.full((B, hkv, kp), -1, np.int32)
    pcnt = np.zeros((B, hkv), np.int32)
    for b, L in enumerate(seqlens):
        for h in range(hkv):
            pool[b, h] = np.sort(rng.choice(L, kp, replace=False))
            pcnt[b, h] = kp
    pool_t, pcnt_t = torch.tensor(pool, device=DEV), torch.tensor(pcnt, device=DEV)
    layers = [make_case(seqlens, hq, hkv, d, "bf16", seed=30 + l) for l in range(4)]
    g = torch.Generator(device="cpu").manual_seed(22)
    news = [(torch.randn((B, hkv, d), generator=g).to(torch.bfloat16).to(DEV),
             torch.randn((B, hkv, d), generator=g).to(torch.bfloat16).to(DEV)) for _ in range(4)]
    ws = ws_for(P, prob, P.OP_REFINE_DECODE, kp, kap)
    res = []
    for overlap in (False, True):
        outs = []
        for l, (q, k, v) in enumerate(layers):
            kc, vc = k.clone(), v.clone()
            idx = torch.zeros((B, hkv, kap), dtype=torch.int32, device=DEV)
            cnt = torch.zeros((B, hkv), dtype=torch.int32, device=DEV)
            out = torch.zeros((B, hq, d), device=DEV)
            outs.append((kc, vc, idx, cnt, out))
        torch.cuda.synchronize()
        for l, (q, k, v) in enumerate(layers):
            kc, vc, idx, cnt, out = outs[l]
            P.refine_decode(prob, q, kc, vc, pool_t, pcnt_t, kp, kap, 0.0883883, idx, cnt, out, ws,
                            k_new=news[l][0], v_new=news[l][1], overlap=overlap and l > 0)
        torch.cuda.synchronize()
        res.append(outs)
    assert P.get_device_status(ws) == 0
    for a, b in zip(res[0], res[1]):
        for x, y in zip(a, b):
            assert torch.equal(x, y)


@pytest.mark.parametrize("kp,kap", [(8192, 2048), (8192, 8191), (3000, 1)])
def test_refine_decode_large_ties(P, kp, kap):
    """All scores equal over pools big enough that every CTA holds more
    first-digit candidates than the ranking buffer: the lowest pool slots win
    on every path, and the attention matches the oracle on that set."""
    seqlens, hq, hkv, d = [40000], 8, 2, 128
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    q, k, v = make_case(seqlens, hq, hkv, d, "bf16", seed=23)
    k[:, :] = k[:, :1]
    pool = torch.arange(0, 4 * kp, 4, dtype=torch.int32, device=DEV).repeat(1, hkv, 1)
    cnt_p = torch.full((1, hkv), kp, dtype=torch.int32, device=DEV)
    idx = torch.zeros((1, hkv, kap), dtype=torch.int32, device=DEV)
    cnt = torch.zeros((1, hkv), dtype=torch.int32, device=DEV)
    out = torch.zeros((1, hq, d), device=DEV)
    ws = ws_for(P, prob, P.OP_REFINE_DECODE, kp, kap)
    P.refine_decode(prob, q, k, v, pool, cnt_p, kp, kap, 0.1, idx, cnt, out, ws)
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    for h in range(hkv):
        assert int(_np(cnt)[0, h]) == kap
        assert np.array_equal(_np(idx)[0, h], np.arange(0, 4 * kap, 4))
    oout, _ = pipeline.attend_layer(q, k, v, [0, 40000], _np(idx), _np(cnt), 0.1)
    assert np.abs(_np(out) - oout).max() <= 2e-3


SELECT_CASES = [
    # (seqlens, Hq, Hkv, d, kappa_p, kappa, keys): the c128k row shape, a
    # ragged batch with an empty and a short sequence, pools of 8192 and 8193
    # members; "int": small integer keys (many exactly equal scores at the
    # threshold, resolved by the lower position: a few per value in the
    # small pool, where they are ranked from the exchanged lists, hundreds in
    # the large one, where the radix digits resolve them); "outlier": one
    # position in 997 has its key row scaled by 512, so the value range is
    # wide and the threshold's window bin crowded (the radix fallback)
    ([131072], 32, 8, 128, 8192, 2048, "normal"),
    ([40000, 9000, 0, 300, 12300], 32, 8, 128, 4096, 1024, "normal"),
    ([30000], 8, 2, 128, 8192, 3000, "normal"),
    ([30000], 8, 2, 128, 8193, 3000, "normal"),
    ([20000, 7000], 32, 8, 128, 8192, 2048, "int"),
    ([2000], 4, 1, 64, 256, 64, "int"),
    ([30000], 8, 2, 128, 8192, 2048, "outlier"),
    ([3000, 5000], 8, 2, 128, 1024, 256, "outlier"),
]


@pytest.mark.parametrize("agg", ["max", "mass"])
@pytest.mark.parametrize("case", SELECT_CASES, ids=lambda c: f"{len(c[0])}seq-kp{c[4]}-k{c[5]}-{c[6]}")
def test_refine_decode_selection_cases(P, case, agg):
    """The fused refined layer's exact top-kappa on the shapes and score
    distributions above, against the oracle, for the maximum over the group
    and for the softmax-mass reading (the MASS instance: sets up to near-ties
    of the fp64 mass); attention on the GPU's set."""
    seqlens, hq, hkv, d, kp, kap, keys = case
    if agg == "mass" and keys == "outlier":
        # outlier logits put every other member's mass far below the fp32
        # range: the GPU's masses tie at zero (lower slot wins) where the
        # fp64 oracle still orders them, so the sets are not comparable
        pytest.skip("masses below the fp32 range")
    B = len(seqlens)
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    q, k, v = make_case(seqlens, hq, hkv, d, "bf16", seed=31)
    if keys == "int":  # small integer keys and queries: exact, often equal, scores
        g = torch.Generator(device="cpu").manual_seed(32)
        k.copy_(torch.randint(-2, 3, k.shape, generator=g).to(k.dtype).to(DEV))
        q.copy_(torch.randint(-1, 2, q.shape, generator=g).to(q.dtype).to(DEV))
    elif keys == "outlier":  # exact in bf16: a power of two
        k[:, ::997] *= 512
    rng = np.random.default_rng(33)
    pool = np.full((B, hkv, kp), -1, np.int32)
    pcnt = np.zeros((B, hkv), np.int32)
    for b, L in enumerate(seqlens):
        for h in range(hkv):
            n = min(kp, L)
            pool[b, h, :n] = np.sort(rng.choice(L, n, replace=False))
            pcnt[b, h] = n
    pool_t, pcnt_t = torch.tensor(pool, device=DEV), torch.tensor(pcnt, device=DEV)
    scale = float(np.float32(1 / math.sqrt(d)))
    ws = ws_for(P, prob, P.OP_REFINE_DECODE, kp, kap)
    i1 = torch.full((B, hkv, kap), -7, dtype=torch.int32, device=DEV)
    c1 = torch.zeros((B, hkv), dtype=torch.int32, device=DEV)
    o1 = torch.full((B, hq, d), 77.0, device=DEV)
    l1 = torch.full((B, hq), 77.0, device=DEV)
    P.refine_decode(prob, q, k, v, pool_t, pcnt_t, kp, kap, scale, i1, c1, o1, ws, lse=l1, mass=agg == "mass")
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    oidx, ocnt, oscores = pipeline.refine_layer(q, k, prob.cu_host.tolist(), pool, pcnt, kap, agg=agg,
                                                softmax_scale=scale)
    gi, gc = _np(i1), _np(c1)
    assert np.array_equal(gc, ocnt)
    for b in range(B):
        for h in range(hkv):
            n, c = int(pcnt[b, h]), int(ocnt[b, h])
            r = dict(zip(pool[b, h, :n].tolist(), oscores[(b, h)].tolist()))
            check_index_set(gi[b, h, :c], oidx[b, h, :c], lambda t: r[t], f"idx b{b} h{h}")
            assert np.all(gi[b, h, c:] == -1)
    oout, _ = pipeline.attend_layer(q, k, v, prob.cu_host.tolist(), gi, gc, scale)
    assert np.abs(_np(o1) - oout).max() <= atol_for("bf16")


# ------------------------------------------------------------------ INT2 keys

@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 128)])
def test_quantize_int2_bit_exact(P, dtype, d):
    seqlens, hq, hkv = [3000, 1], 8, 2
    prob = problem(P, seqlens, hq, hkv, d, dtype)
    _, k, _ = make_case(seqlens, hq, hkv, d, dtype, seed=24, scale_rows=True)
    k[0, 5] = 0.0            # a constant (zero) row: step 0
    k[1, 9, :32] = -0.0      # signed zeros in one group
    k[1, 9, 32:64] = 3.0
    T = prob.total_tokens
    codes = torch.full((hkv, T, d // 4), 0xAB, dtype=torch.uint8, device=DEV)
    params = torch.full((hkv, T, d // 32, 2), -1, dtype=torch.int16, device=DEV)
    ws = ws_for(P, prob, P.OP_QUANTIZE)
    P.quantize_k_int2(prob, k, codes, params, ws=ws)
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    oc, op = oracle.quantize_int2_rows(_np(k).reshape(hkv * T, d))
    assert np.array_equal(codes.cpu().numpy().reshape(hkv * T, d // 4), oc)
    assert np.array_equal(params.cpu().numpy().view(np.uint16).reshape(hkv * T, d // 32, 2), op)
    # only the listed rows change when tok_rows is given
    rows = torch.tensor([0, 2999], dtype=torch.int32, device=DEV)
    codes2 = torch.zeros_like(codes)
    params2 = torch.zeros_like(params)
    P.quantize_k_int2(prob, k, codes2, params2, tok_rows=rows, ws=ws)
    torch.cuda.synchronize()
    c2 = codes2.cpu().numpy()
    assert np.array_equal(c2[:, [0, 2999]], codes.cpu().numpy()[:, [0, 2999]])
    assert not c2[:, 1:2999].any()


INT2_CASES = [
    ([8192], 32, 8, 2048),
    ([5000, 1031, 0, 300], 8, 2, 1024),
    ([40000], 16, 4, 4096),
    ([1024, 1025], 8, 2, 1024),
    ([3000, 129], 16, 8, 500),   # G = 2
    ([2500], 64, 8, 700),        # G = 8 (two head quads)
]


@pytest.mark.parametrize("case", INT2_CASES, ids=lambda c: f"{c[0]}-{c[1]}/{c[2]}-kp{c[3]}")
def test_propose_int2_vs_oracle(P, case):
    seqlens, hq, hkv, kp = case
    d = 128
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    q, k, _ = make_case(seqlens, hq, hkv, d, "bf16", seed=25)
    T = prob.total_tokens
    codes = torch.zeros((hkv, T, d // 4), dtype=torch.uint8, device=DEV)
    params = torch.zeros((hkv, T, d // 32, 2), dtype=torch.int16, device=DEV)
    P.quantize_k_int2(prob, k, codes, params)
    pool = torch.full((len(seqlens), hkv, kp), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((len(seqlens), hkv), -7, dtype=torch.int32, device=DEV)
    ws = ws_for(P, prob, P.OP_PROPOSE, kp)
    P.propose_int2(prob, q, codes, params, kp, pool, cnt, ws)
    torch.cuda.synchronize()
    assert P.get_device_status(ws) == 0
    gscores = _np(ws[256:256 + hkv * T * 4].view(torch.float32)).reshape(hkv, T)
    opool, ocnt, oscores = pipeline.propose_layer_int2(q, codes.cpu().numpy(), params.cpu().numpy().view(np.uint16),
                                                       prob.cu_host.tolist(), kp)
    gp, gc = _np(pool), _np(cnt)
    assert np.array_equal(gc, ocnt)
    cu = prob.cu_host
    pr = params.cpu().numpy().view(np.uint16).view(np.float16).astype(np.float64)  # [Hkv][T][4][2]
    qf = _np(q).astype(np.float64)
    G = hq // hkv
    for b in range(len(seqlens)):
        for h in range(hkv):
            s = oscores[(b, h)]
            n = int(ocnt[b, h])
            if n:
                gs = gscores[h, cu[b]:cu[b + 1]]
                # A score is a sum of the products S * D and L * Q, which may cancel,
                # and each side sums D = q . c over a group in its own order.  The
                # forward error of such sums is bounded by a few dozen units in the
                # last place of the sum of the terms' magnitudes (R16), not of the
                # score: |S| 3 sum|q| + |L| |Q| per group, the largest over the heads.
                qg = qf[b, h * G:(h + 1) * G].reshape(G, 4, 32)
                sa, qa = np.abs(qg).sum(axis=2), np.abs(qg.sum(axis=2))  # [G][4]
                S, Lz = np.abs(pr[h, cu[b]:cu[b + 1], :, 0]), np.abs(pr[h, cu[b]:cu[b + 1], :, 1])
                bound = (S[:, None, :] * 3 * sa[None] + Lz[:, None, :] * qa[None]).sum(axis=2).max(axis=1)
                assert np.all(np.abs(gs - s) <= 64 * 2.0 ** -24 * bound), (b, h)
            check_index_set(gp[b, h, :n], opool[b, h, :n], lambda t: s[t], f"int2 pool b{b} h{h}")
            assert np.all(gp[b, h, n:] == -1)


def test_propose_int2_unsupported_shapes(P):
    prob = problem(P, [1000], 8, 2, 64, "bf16")
    q, k, _ = make_case([1000], 8, 2, 64, "bf16", seed=26)
    codes = torch.zeros((2, 1000, 16), dtype=torch.uint8, device=DEV)
    params = torch.zeros((2, 1000, 2, 2), dtype=torch.int16, device=DEV)
    pool = torch.zeros((1, 2, 100), dtype=torch.int32, device=DEV)
    cnt = torch.zeros((1, 2), dtype=torch.int32, device=DEV)
    with pytest.raises(P.PrismError) as e:
        P.propose_int2(prob, q, codes, params, 100, pool, cnt, ws_for(P, prob, P.OP_PROPOSE, 100))
    assert e.value.status == P.ERR_UNSUPPORTED


# ------------------------------------------------------------------ selection granularity

SETS_CASES = [
    # (seqlens, Hq, Hkv, d, kappa_p, kappa): ragged with an empty and a short
    # sequence (pools and sets shorter than their budgets), one KV head, G = 1
    ([5000, 0, 700, 2500], 32, 8, 128, 1024, 256),
    ([3000], 4, 1, 64, 512, 100),
    ([1500, 4000], 8, 8, 128, 600, 600),
]


@pytest.mark.parametrize("case", SETS_CASES, ids=lambda c: f"{len(c[0])}seq-{c[1]}/{c[2]}-kp{c[4]}")
@pytest.mark.parametrize("sets", ["q_head", "sequence"])
def test_selection_granularity_calls_vs_oracle(P, case, sets):
    seqlens, hq, hkv, d, kp, kap = case
    B = len(seqlens)
    prob = problem(P, seqlens, hq, hkv, d, "bf16")
    q, k, v = make_case(seqlens, hq, hkv, d, "bf16", seed=41)
    cu = prob.cu_host.tolist()
    code = P.SETS_Q_HEAD if sets == "q_head" else P.SETS_SEQUENCE
    kq = torch.zeros(k.shape, dtype=torch.int8, device=DEV)
    sc = torch.zeros(k.shape[:2], dtype=torch.float32, device=DEV)
    P.quantize_k(prob, k, kq, sc)
    prow = 1 if sets == "sequence" else hkv
    srow = hq if sets == "q_head" else 1
    pool = torch.full((B, prow, kp), -7, dtype=torch.int32, device=DEV)
    pcnt = torch.zeros((B, prow), dtype=torch.int32, device=DEV)
    wp = ws_for(P, prob, P.OP_PROPOSE, kp)
    P.propose_ex(prob, q, kq, sc, kp, pool, pcnt, code, wp)
    idx = torch.full((B, srow, kap), -7, dtype=torch.int32, device=DEV)
    cnt = torch.zeros((B, srow), dtype=torch.int32, device=DEV)
    wr = ws_for(P, prob, P.OP_REFINE, kp, kap)
    P.refine_ex(prob, q, k, pool, pcnt, kp, kap, idx, cnt, code, wr)
    out = torch.full((B, hq, d), 77.0, device=DEV)
    lse = torch.full((B, hq), 77.0, device=DEV)
    wd = ws_for(P, prob, P.OP_SPARSE_DECODE, 0, kap)
    scale = float(np.float32(1 / math.sqrt(d)))
    P.sparse_decode_ex(prob, q, k, v, idx, cnt, kap, scale, code, out, wd, lse=lse)
    torch.cuda.synchronize()
    for w in (wp, wr, wd):
        assert P.get_device_status(w) == 0
    okq, osc = pipeline.quantize_layer(k)
    gp, gpc, gi, gc = _np(pool), _np(pcnt), _np(idx), _np(cnt)
    if sets == "sequence":
        opool, ocnt, oscore = pipeline.propose_layer_seq(q, okq, osc, cu, kp)
        for b in range(B):
            n = int(ocnt[b])
            assert int(gpc[b, 0]) == n == min(kp, seqlens[b])
            check_index_set(gp[b, 0, :n], opool[b, :n], lambda t: oscore[b][t], f"pool {b}")
            assert np.all(gp[b, 0, n:] == -1)
        oidx, oc, orr = pipeline.refine_layer_seq(q, k, cu, gp[:, 0], gpc[:, 0], kap)
        for b in range(B):
            n, c = int(gpc[b, 0]), int(oc[b])
            assert int(gc[b, 0]) == c
            r = dict(zip(gp[b, 0, :n].tolist(), orr[b].tolist()))
            check_index_set(gi[b, 0, :c], oidx[b, :c], lambda t: r[t], f"idx {b}")
            assert np.all(gi[b, 0, c:] == -1)
        oout, olse = pipeline.attend_layer_sets(q, k, v, cu, gi[:, 0], gc[:, 0], "sequence", scale)
    else:
        opool, ocnt, oscore = pipeline.propose_layer(q, okq, osc, cu, kp)
        assert np.array_equal(gpc, ocnt)
        oidx, oc, orr = pipeline.refine_layer_heads(q, k, cu, gp, gpc, kap)
        G = hq // hkv
        for b in range(B):
            for h in range(hq):
                n, c = int(gpc[b, h // G]), int(oc[b, h])
                assert int(gc[b, h]) == c
                r = dict(zip(gp[b, h // G, :n].tolist(), orr[(b, h)].tolist()))
                check_index_set(gi[b, h, :c], oidx[b, h, :c], lambda t: r[t], f"idx {b},{h}")
                assert np.all(gi[b, h, c:] == -1)
        oout, olse = pipeline.attend_layer_sets(q, k, v, cu, gi, gc, "q_head", scale)
    tol = atol_for("bf16")
    assert np.abs(_np(out) - oout).max() <= tol
    gl = _np(lse)
    fin = np.isfinite(olse)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.abs(gl[fin] - olse[fin]).max() <= 10 * tol

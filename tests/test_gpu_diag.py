"""The index-overlap entry point and the cross-layer overlap diagnostic
(Prism Attention, sec. 3 "Observations", Figures 1 and 12) against the
oracle's set intersection and brute force."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_top_proposal_b200 import diagnostics, workload
from oracle import pipeline
from parity_util import check_index_set

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _sets(rng, rows, stride, L):
    a = np.full((rows, stride), -1, np.int32)
    c = np.zeros(rows, np.int32)
    for r in range(rows):
        n = int(rng.integers(0, min(stride, L) + 1))
        a[r, :n] = np.sort(rng.choice(L, n, replace=False))
        c[r] = n
    return a, c


def test_index_overlap_matches_oracle(prism_lib):
    P = prism_lib
    rng = np.random.default_rng(5)
    for rows, sa, sb, L in [(1, 1, 1, 1), (7, 64, 300, 500), (40, 2048, 8192, 131072), (3, 5, 5, 5)]:
        a, ca = _sets(rng, rows, sa, L)
        b, cb = _sets(rng, rows, sb, L)
        if rows == 3:
            ca[1] = sa + 9  # a count above the stride is clamped
            cb[2] = -4      # a negative count is empty
        out = torch.full((rows,), -1, dtype=torch.int32, device=DEV)
        P.index_overlap(torch.tensor(a, device=DEV), torch.tensor(ca, device=DEV),
                        torch.tensor(b, device=DEV), torch.tensor(cb, device=DEV), out)
        got = out.cpu().numpy()
        for r in range(rows):
            na, nb = min(max(ca[r], 0), sa), min(max(cb[r], 0), sb)
            assert got[r] == oracle.set_overlap(a[r, :na], b[r, :nb]), (rows, r)


def test_overlap_diagnostic_c8k(prism_lib):
    """Exact top-kappa per layer against the oracle's exact selection over
    every position; the offset table against set intersections on the host."""
    res = diagnostics.run("c8k", max_offset=3)
    cfg = workload.config("c8k")
    layers = list(workload.generate(cfg, DEV))
    dec_p = prism_lib.Problem(cfg.seqlens, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim,
                              prism_lib.BF16, device=DEV)
    qs, ks = [x.q for x in layers], [x.k for x in layers]
    exact = diagnostics.exact_topk_sets(dec_p, qs, ks, cfg.kappa)
    L = cfg.seqlens[0]
    allpos = np.arange(L, dtype=np.int32)
    sets = []
    for l, (idx, cnt) in enumerate(exact):
        gi = idx.cpu().numpy()
        per = []
        for h in range(cfg.num_kv_heads):
            G = cfg.G
            q = layers[l].q[0, h * G:(h + 1) * G].float().cpu().numpy()
            k = layers[l].k[h].float().cpu().numpy()
            oi, r = oracle.refine_row(q, k, allpos, cfg.kappa)
            check_index_set(gi[0, h], oi, lambda t: r[t], f"exact L{l} h{h}")
            per.append(set(gi[0, h].tolist()))
        sets.append(per)
    for o in range(1, 4):
        want = np.mean([len(sets[l][h] & sets[l + o][h]) / cfg.kappa
                        for l in range(cfg.num_layers - o) for h in range(cfg.num_kv_heads)])
        assert abs(res["static_overlap"][o - 1] - want) < 1e-12, o
        assert 0.0 <= res["static_overlap"][o - 1] <= res["pool_coverage"][o - 1] <= 1.0
    assert all(0.0 <= x <= 1.0 for x in res["prism_recall_per_layer"])

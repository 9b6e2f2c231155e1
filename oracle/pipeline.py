"""Layer- and step-level drivers of the CPU oracle (test infrastructure).

Packed layouts, shared with the CUDA library's interface:
  q        [B][Hq][d]
  K, V     [Hkv][T][d]   rows of sequence b at cu_seqlens[b] .. cu_seqlens[b+1]
  kq       [Hkv][T][d]   int8,  k_scale [Hkv][T] fp32
  pool     [B][Hkv][kappa_p] int32 positions within the sequence, ascending,
           -1 past pool_cnt[b][h]
  idx      [B][Hkv][kappa]   same convention, cnt[b][h]
  out      [B][Hq][d] fp32,  lse [B][Hq] fp32
Query head hq reads KV head hq // G.  Each (sequence, KV head) row is
independent, so every function loops over rows and calls the C oracle.

The layer schedule (Prism Attention, sec. 5.3 "Accuracy-efficiency
trade-off": in "g x" one layer in every x is a proposal layer) is read as
``layer % group == 0``; the pool of the latest proposal layer serves every
layer up to the next one.  A proposal layer also refines its own pool with
exact scores and attends over the refined set, so every layer attends over
kappa exactly rescored tokens (reading of sec. 6: refined layers re-select
their own top-kappa inside the proposed region).
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional

import numpy as np

from . import (attend, pool_topk, propose_row, propose_row_int2, propose_row_seq, quantize_int2_rows,
               quantize_rows, refine_row, refine_row_heads, refine_row_mass, refine_row_seq)


def _np(x):
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").float().numpy() if x.dtype != torch.int8 and \
                x.dtype != torch.int32 and x.dtype != torch.int64 else x.detach().to("cpu").numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x)


def quantize_layer(k):
    """kq [Hkv][T][d] int8, scale [Hkv][T] fp32 from K [Hkv][T][d]."""
    k = _np(k).astype(np.float32)
    Hkv, T, d = k.shape
    kq, sc = quantize_rows(k.reshape(Hkv * T, d))
    return kq.reshape(Hkv, T, d), sc.reshape(Hkv, T)


def propose_layer(q, kq, scale, cu, kappa_p: int, rows=None, agg: str = "max"):
    """pool [B][Hkv][kappa_p] (-1 padded), pool_cnt [B][Hkv], scores per row
    (agg: how the group's query heads combine, "max" or "sum")."""
    q = _np(q).astype(np.float32)
    kq, scale = _np(kq), _np(scale).astype(np.float32)
    B, Hq, d = q.shape
    Hkv = kq.shape[0]
    G = Hq // Hkv
    pool = np.full((B, Hkv, kappa_p), -1, np.int32)
    cnt = np.zeros((B, Hkv), np.int32)
    scores: Dict = {}
    for b in range(B):
        t0, t1 = cu[b], cu[b + 1]
        for h in range(Hkv):
            if rows is not None and (b, h) not in rows:
                continue
            p, s = propose_row(q[b, h * G:(h + 1) * G], kq[h, t0:t1], scale[h, t0:t1], kappa_p, agg)
            pool[b, h, :p.size] = p
            cnt[b, h] = p.size
            scores[(b, h)] = s
    return pool, cnt, scores


def quantize_layer_int2(k):
    """INT2 codes [Hkv][T][d/4] uint8 and params [Hkv][T][d/32][2] (fp16 bits)."""
    k = _np(k).astype(np.float32)
    Hkv, T, d = k.shape
    codes, params = quantize_int2_rows(k.reshape(Hkv * T, d))
    return codes.reshape(Hkv, T, d // 4), params.reshape(Hkv, T, d // 32, 2)


def propose_layer_int2(q, codes, params, cu, kappa_p: int, rows=None):
    """INT2 proposal: pool [B][Hkv][kappa_p] (-1 padded), pool_cnt, scores per row."""
    q = _np(q).astype(np.float32)
    codes, params = _np(codes), _np(params)
    B, Hq, d = q.shape
    Hkv = codes.shape[0]
    G = Hq // Hkv
    pool = np.full((B, Hkv, kappa_p), -1, np.int32)
    cnt = np.zeros((B, Hkv), np.int32)
    scores: Dict = {}
    for b in range(B):
        t0, t1 = cu[b], cu[b + 1]
        for h in range(Hkv):
            if rows is not None and (b, h) not in rows:
                continue
            p, sc = propose_row_int2(q[b, h * G:(h + 1) * G], codes[h, t0:t1],
                                            params[h, t0:t1], kappa_p)
            pool[b, h, :p.size] = p
            cnt[b, h] = p.size
            scores[(b, h)] = sc
    return pool, cnt, scores


def refine_layer(q, k, cu, pool, pool_cnt, kappa: int, rows=None, agg: str = "max",
                 softmax_scale: Optional[float] = None):
    """idx [B][Hkv][kappa] (-1 padded), cnt [B][Hkv], exact pool scores per row
    (agg as in propose_layer, or "mass": the group's softmax mass over the
    pool at softmax_scale, default 1/sqrt(d))."""
    q = _np(q).astype(np.float32)
    k = _np(k).astype(np.float32)
    pool, pool_cnt = _np(pool), _np(pool_cnt)
    B, Hq, d = q.shape
    Hkv = k.shape[0]
    G = Hq // Hkv
    idx = np.full((B, Hkv, kappa), -1, np.int32)
    cnt = np.zeros((B, Hkv), np.int32)
    scores: Dict = {}
    for b in range(B):
        t0, t1 = cu[b], cu[b + 1]
        for h in range(Hkv):
            if rows is not None and (b, h) not in rows:
                continue
            n = int(pool_cnt[b, h])
            if agg == "mass":
                sc = float(np.float32(1.0 / math.sqrt(d))) if softmax_scale is None else softmax_scale
                sel, r = refine_row_mass(q[b, h * G:(h + 1) * G], k[h, t0:t1], pool[b, h, :n], kappa, sc)
            else:
                sel, r = refine_row(q[b, h * G:(h + 1) * G], k[h, t0:t1], pool[b, h, :n], kappa, agg)
            idx[b, h, :sel.size] = sel
            cnt[b, h] = sel.size
            scores[(b, h)] = r
    return idx, cnt, scores


def pool_topk_layer(scores, pool, pool_cnt, kappa: int, rows=None):
    """The proposal layer's own set from its quantized scores (the
    alternative to exact rescoring): scores[(b, h)] are the proposal scores
    of propose_layer; idx [B][Hkv][kappa] (-1 padded), cnt [B][Hkv]."""
    pool, pool_cnt = _np(pool), _np(pool_cnt)
    B, Hkv = pool_cnt.shape
    idx = np.full((B, Hkv, kappa), -1, np.int32)
    cnt = np.zeros((B, Hkv), np.int32)
    for b in range(B):
        for h in range(Hkv):
            if rows is not None and (b, h) not in rows:
                continue
            n = int(pool_cnt[b, h])
            sel = pool_topk(scores[(b, h)], pool[b, h, :n], kappa)
            idx[b, h, :sel.size] = sel
            cnt[b, h] = sel.size
    return idx, cnt


def propose_layer_seq(q, kq, scale, cu, kappa_p: int):
    """One pool per sequence shared by every head: pool [B][kappa_p] (-1
    padded), pool_cnt [B], head-max proposal scores per sequence."""
    q = _np(q).astype(np.float32)
    kq, scale = _np(kq), _np(scale).astype(np.float32)
    B = q.shape[0]
    pool = np.full((B, kappa_p), -1, np.int32)
    cnt = np.zeros((B,), np.int32)
    scores: Dict = {}
    for b in range(B):
        t0, t1 = cu[b], cu[b + 1]
        p, s = propose_row_seq(q[b], kq[:, t0:t1], scale[:, t0:t1], kappa_p)
        pool[b, :p.size] = p
        cnt[b] = p.size
        scores[b] = s
    return pool, cnt, scores


def refine_layer_seq(q, k, cu, pool, pool_cnt, kappa: int):
    """One set per sequence from its pool: idx [B][kappa], cnt [B], head-max
    exact pool scores per sequence."""
    q = _np(q).astype(np.float32)
    k = _np(k).astype(np.float32)
    pool, pool_cnt = _np(pool), _np(pool_cnt)
    B = q.shape[0]
    idx = np.full((B, kappa), -1, np.int32)
    cnt = np.zeros((B,), np.int32)
    scores: Dict = {}
    for b in range(B):
        t0, t1 = cu[b], cu[b + 1]
        n = int(pool_cnt[b])
        sel, r = refine_row_seq(q[b], k[:, t0:t1], pool[b, :n], kappa)
        idx[b, :sel.size] = sel
        cnt[b] = sel.size
        scores[b] = r
    return idx, cnt, scores


def refine_layer_heads(q, k, cu, pool, pool_cnt, kappa: int, rows=None):
    """One set per query head over its group's pool: idx [B][Hq][kappa], cnt
    [B][Hq], exact per-head pool scores keyed (b, hq)."""
    q = _np(q).astype(np.float32)
    k = _np(k).astype(np.float32)
    pool, pool_cnt = _np(pool), _np(pool_cnt)
    B, Hq, d = q.shape
    Hkv = k.shape[0]
    G = Hq // Hkv
    idx = np.full((B, Hq, kappa), -1, np.int32)
    cnt = np.zeros((B, Hq), np.int32)
    scores: Dict = {}
    for b in range(B):
        t0, t1 = cu[b], cu[b + 1]
        for h in range(Hkv):
            if rows is not None and (b, h) not in rows:
                continue
            n = int(pool_cnt[b, h])
            sel, r = refine_row_heads(q[b, h * G:(h + 1) * G], k[h, t0:t1], pool[b, h, :n], kappa)
            for g in range(G):
                idx[b, h * G + g, :sel.shape[1]] = sel[g]
                cnt[b, h * G + g] = sel.shape[1]
                scores[(b, h * G + g)] = r[g]
    return idx, cnt, scores


def attend_layer_sets(q, k, v, cu, idx, cnt, sets: str, softmax_scale: Optional[float] = None):
    """Attention of every query head over its set: sets "q_head" (idx
    [B][Hq][kappa]) or "sequence" (idx [B][kappa], shared by every head)."""
    q = _np(q).astype(np.float32)
    k = _np(k).astype(np.float32)
    v = _np(v).astype(np.float32)
    idx, cnt = _np(idx), _np(cnt)
    B, Hq, d = q.shape
    Hkv = k.shape[0]
    G = Hq // Hkv
    if softmax_scale is None:
        softmax_scale = float(np.float32(1.0 / math.sqrt(d)))
    out = np.zeros((B, Hq, d), np.float32)
    lse = np.full((B, Hq), -np.inf, np.float32)
    for b in range(B):
        t0, t1 = cu[b], cu[b + 1]
        for hq in range(Hq):
            h = hq // G
            sel = idx[b, hq, :int(cnt[b, hq])] if sets == "q_head" else idx[b, :int(cnt[b])]
            out[b, hq], lse[b, hq] = attend(q[b, hq], k[h, t0:t1], v[h, t0:t1], sel, softmax_scale)
    return out, lse


def attend_layer(q, k, v, cu, idx, cnt, softmax_scale: Optional[float] = None, rows=None):
    """Sparse attention over idx (idx None = dense over every position)."""
    q = _np(q).astype(np.float32)
    k = _np(k).astype(np.float32)
    v = _np(v).astype(np.float32)
    B, Hq, d = q.shape
    Hkv = k.shape[0]
    G = Hq // Hkv
    if softmax_scale is None:
        softmax_scale = float(np.float32(1.0 / math.sqrt(d)))
    out = np.zeros((B, Hq, d), np.float32)
    lse = np.full((B, Hq), -np.inf, np.float32)
    for b in range(B):
        t0, t1 = cu[b], cu[b + 1]
        for h in range(Hkv):
            if rows is not None and (b, h) not in rows:
                continue
            sel = None if idx is None else _np(idx)[b, h, :int(_np(cnt)[b, h])]
            for g in range(G):
                hq = h * G + g
                out[b, hq], lse[b, hq] = attend(q[b, hq], k[h, t0:t1], v[h, t0:t1], sel,
                                                softmax_scale)
    return out, lse


def decode_step(cfg, layers, rows=None, proposal_select: str = "exact") -> List[dict]:
    """One decode step over the given layers (workload.Layer objects, in order).

    Returns, per layer: kq/scale (proposal layers), pool/pool_cnt (from the
    latest proposal layer), idx/cnt, out/lse.  proposal_select: "exact" (a
    proposal layer refines its own pool, the default reading) or "quantized"
    (it takes the top kappa of its pool by its proposal scores).
    """
    cu = cfg.cu_seqlens
    res = []
    pool = pool_cnt = None
    for lay in layers:
        r = {"layer": lay.index}
        proposal = cfg.is_proposal(lay.index)
        if proposal:
            kq, sc = quantize_layer(lay.k)
            pool, pool_cnt, pscores = propose_layer(lay.q, kq, sc, cu, cfg.kappa_p, rows)
            r["kq"], r["scale"] = kq, sc
        assert pool is not None, "the first layer of a step must be a proposal layer"
        r["pool"], r["pool_cnt"] = pool, pool_cnt
        if proposal and proposal_select == "quantized":
            idx, cnt = pool_topk_layer(pscores, pool, pool_cnt, cfg.kappa, rows)
        else:
            idx, cnt, _ = refine_layer(lay.q, lay.k, cu, pool, pool_cnt, cfg.kappa, rows)
        r["idx"], r["cnt"] = idx, cnt
        r["out"], r["lse"] = attend_layer(lay.q, lay.k, lay.v, cu, idx, cnt, rows=rows)
        res.append(r)
    return res

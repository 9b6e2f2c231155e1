"""Cross-layer index overlap on generated workloads (Prism Attention, sec. 3
"Observations", Figure 1 and Figure 12).

For each layer l of a decode step the exact top-kappa set (every position
scored with the exact keys, no proposal) is found with prism_refine over a
pool of all positions.  Then, for layer offsets o = 1 .. max_offset:

  static_overlap[o]  mean over rows and layer pairs (l, l + o) of
                     |top_kappa(l) & top_kappa(l + o)| / |top_kappa(l + o)|
                     -- how well a set reused from layer l serves layer l + o
                     (Figure 1);
  pool_coverage[o]   the same with the expanded top-(rho kappa) set of layer l
                     in place of top_kappa(l) -- the coverage an expanded
                     proposal region keeps (Figure 12, right panels);

and, for the decoder's own sets, prism_recall[l] = |idx(l) & top_kappa(l)| /
|top_kappa(l)|, the share of the exact top-kappa that the proposal-refined
selection recovers.  Intersections are counted on the GPU
(prism_index_overlap); rows are (sequence, KV head) pairs, as the selection.
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import torch

from . import prism


def exact_topk_sets(p: prism.Problem, qs: Sequence, ks: Sequence, kappa: int, stream=None):
    """Per layer: (idx [B][Hkv][kappa], cnt [B][Hkv]) of the exact top-kappa
    over every position (prism_refine on the pool of all positions)."""
    B, Hkv = p.shape.batch, p.shape.num_kv_heads
    L = max(p.seqlens) if p.seqlens else 0
    dev = p.cu_dev.device
    kp = max(L, kappa)
    pool = torch.full((B, Hkv, kp), -1, dtype=torch.int32, device=dev)
    pcnt = torch.zeros((B, Hkv), dtype=torch.int32, device=dev)
    for b, Lb in enumerate(p.seqlens):
        pool[b, :, :Lb] = torch.arange(Lb, dtype=torch.int32, device=dev)
        pcnt[b, :] = Lb
    ws = torch.zeros(prism.workspace_size(p, prism.OP_REFINE, kp, kappa), dtype=torch.uint8, device=dev)
    out = []
    for q, k in zip(qs, ks):
        idx = torch.full((B, Hkv, kappa), -1, dtype=torch.int32, device=dev)
        cnt = torch.zeros((B, Hkv), dtype=torch.int32, device=dev)
        prism.refine(p, q, k, pool, pcnt, kp, kappa, idx, cnt, ws, stream=stream)
        out.append((idx, cnt))
    return out


def overlap_counts(a, cnt_a, b, cnt_b) -> torch.Tensor:
    out = torch.empty(cnt_a.numel(), dtype=torch.int32, device=cnt_a.device)
    prism.index_overlap(a.reshape(cnt_a.numel(), -1), cnt_a.reshape(-1), b.reshape(cnt_b.numel(), -1),
                        cnt_b.reshape(-1), out)
    return out


def _ratio(hits: torch.Tensor, denom: torch.Tensor) -> float:
    d = denom.reshape(-1).double()
    keep = d > 0
    return float((hits.double()[keep] / d[keep]).mean()) if bool(keep.any()) else float("nan")


def overlap_by_offset(sets: List, wide: List, max_offset: int) -> Dict[str, List[float]]:
    """sets[l] = (idx, cnt) top-kappa per layer, wide[l] the expanded
    top-(rho kappa) sets; means over rows and layer pairs per offset."""
    n = len(sets)
    static, cover = [], []
    for o in range(1, max_offset + 1):
        s_r, c_r = [], []
        for l in range(n - o):
            ia, ca = sets[l]
            ib, cb = sets[l + o]
            s_r.append(_ratio(overlap_counts(ib, cb, ia, ca), cb))
            wa, wc = wide[l]
            c_r.append(_ratio(overlap_counts(ib, cb, wa, wc), cb))
        static.append(sum(s_r) / len(s_r) if s_r else float("nan"))
        cover.append(sum(c_r) / len(c_r) if c_r else float("nan"))
    return {"static_overlap": static, "pool_coverage": cover}


def recall(dec_sets: List, exact: List) -> List[float]:
    """Per layer, the share of the exact top-kappa that the decoder's sets hold."""
    return [_ratio(overlap_counts(e[0], e[1], d[0], d[1]), e[1]) for d, e in zip(dec_sets, exact)]


def run(config: str = "c8k", max_offset: int = 7, rho: int = 0, device="cuda") -> dict:
    """The overlap table of one generated workload: exact top-kappa and
    top-(rho kappa) sets per layer, their offsets, and the recall of one
    decode step of the proposal-refined path (rho defaults to the workload's
    kappa_p / kappa)."""
    from . import workload
    from .decoder import PrismDecoder

    cfg = workload.config(config)
    dt = prism.BF16 if cfg.dtype == "bf16" else prism.F32
    rho = rho or cfg.kappa_p // cfg.kappa
    layers = list(workload.generate(cfg, device))
    qs, ks, vs = [x.q for x in layers], [x.k for x in layers], [x.v for x in layers]
    dec = PrismDecoder(cfg.seqlens, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, dt,
                       cfg.num_layers, cfg.group, cfg.kappa_p, cfg.kappa, device=device)
    kqs, scs = {}, {}
    for l in cfg.proposal_layers:
        kqs[l] = torch.empty(ks[l].shape, dtype=torch.int8, device=device)
        scs[l] = torch.empty(ks[l].shape[:2], dtype=torch.float32, device=device)
        prism.quantize_k(dec.p, ks[l], kqs[l], scs[l])
    dec.step(qs, ks, vs, kqs, scs)
    exact = exact_topk_sets(dec.p, qs, ks, cfg.kappa)
    wide = exact_topk_sets(dec.p, qs, ks, rho * cfg.kappa)
    tab = overlap_by_offset(exact, wide, min(max_offset, cfg.num_layers - 1))
    rec = recall(list(zip(dec.idx, dec.cnt)), exact)
    return {"workload": cfg.name, "kappa": cfg.kappa, "rho": rho, "offsets": list(range(1, len(tab["static_overlap"]) + 1)),
            **tab, "prism_recall_per_layer": rec, "prism_recall_mean": sum(rec) / len(rec)}


if __name__ == "__main__":
    import argparse
    import json

    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--config", default="c8k")
    ap.add_argument("--max-offset", type=int, default=7)
    ap.add_argument("--rho", type=int, default=0)
    a = ap.parse_args()
    print(json.dumps(run(a.config, a.max_offset, a.rho)))

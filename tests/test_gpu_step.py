"""Whole decode steps through the layer driver vs the oracle.

Small configurations are checked on every (sequence, KV head) row of every
layer.  The full-size configurations run the call sequence the benchmark
times (captured step graph, the token's rows appended inside the kernels,
overlapped refined layers) and are checked on every row of a whole proposal
group; a second test samples rows of a step whose caches already hold the
token (no appends).
Each stage is checked on the GPU's own upstream set (cascade control).
"""
import math

import numpy as np
import pytest
import torch

from kv_cache_top_proposal_b200 import workload
from kv_cache_top_proposal_b200.decoder import PrismDecoder
from oracle import pipeline
from parity_util import atol_for, check_index_set

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _np(t):
    return t.detach().float().cpu().numpy() if t.dtype not in (torch.int32, torch.int8) \
        else t.detach().cpu().numpy()


def _decoder(P, cfg, fused=True, group_agg="max"):
    return PrismDecoder(cfg.seqlens, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim,
                        P.F32 if cfg.dtype == "f32" else P.BF16, cfg.num_layers, cfg.group,
                        cfg.kappa_p, cfg.kappa, device=DEV, fused=fused, group_agg=group_agg)


def _prefill_kq(P, dec, cfg, lay):
    kq = torch.zeros(lay.k.shape, dtype=torch.int8, device=DEV)
    sc = torch.zeros(lay.k.shape[:2], dtype=torch.float32, device=DEV)
    P.quantize_k(dec.p, lay.k, kq, sc)
    return kq, sc


def _check_layer(dec, cfg, l, lay, kq, sc, rows, agg="max"):
    cu = cfg.cu_seqlens
    src = l - l % cfg.group
    gpool, gpc = _np(dec.pool[src]), _np(dec.pool_cnt[src])
    if l == src:
        pagg = "max" if agg == "mass" else agg  # the mass reading leaves the proposal at the max
        opool, ocnt, osc = pipeline.propose_layer(lay.q, kq, sc, cu, cfg.kappa_p, rows=rows, agg=pagg)
        for (b, h) in rows:
            n = int(ocnt[b, h])
            assert int(gpc[b, h]) == n
            check_index_set(gpool[b, h, :n], opool[b, h, :n], lambda t: osc[(b, h)][t],
                            f"L{l} pool {b},{h}")
            assert np.all(gpool[b, h, n:] == -1)
    gidx, gcnt = _np(dec.idx[l]), _np(dec.cnt[l])
    oidx, ocnt, orr = pipeline.refine_layer(lay.q, lay.k, cu, gpool, gpc, cfg.kappa, rows=rows, agg=agg)
    for (b, h) in rows:
        n = int(gpc[b, h])
        r = dict(zip(gpool[b, h, :n].tolist(), orr[(b, h)].tolist()))
        c = int(ocnt[b, h])
        assert int(gcnt[b, h]) == c
        check_index_set(gidx[b, h, :c], oidx[b, h, :c], lambda t: r[t], f"L{l} idx {b},{h}")
        assert set(gidx[b, h, :c].tolist()) <= set(gpool[b, h, :n].tolist())
    oout, olse = pipeline.attend_layer(lay.q, lay.k, lay.v, cu, gidx, gcnt, dec.scale, rows=rows)
    gout, glse = _np(dec.out[l]), _np(dec.lse[l])
    G = cfg.G
    tol = atol_for(cfg.dtype)
    for (b, h) in rows:
        sl = slice(h * G, (h + 1) * G)
        assert np.abs(gout[b, sl] - oout[b, sl]).max() <= tol, (l, b, h)
        assert np.abs(glse[b, sl] - olse[b, sl]).max() <= 10 * tol, (l, b, h)


def _all_rows(cfg):
    return [(b, h) for b in range(cfg.batch) for h in range(cfg.num_kv_heads)]


def _invariants(dec, cfg, l):
    src = l - l % cfg.group
    gp, gpc = _np(dec.pool[src]), _np(dec.pool_cnt[src])
    gi, gc = _np(dec.idx[l]), _np(dec.cnt[l])
    for b, L in enumerate(cfg.seqlens):
        for h in range(cfg.num_kv_heads):
            n, c = int(gpc[b, h]), int(gc[b, h])
            assert n == min(cfg.kappa_p, L) and c == min(cfg.kappa, n)
            p, i = gp[b, h, :n], gi[b, h, :c]
            assert np.all(np.diff(p) > 0) and (n == 0 or (p[0] >= 0 and p[-1] < L))
            assert np.all(np.diff(i) > 0) and np.all(np.isin(i, p))
    assert np.all(np.isfinite(_np(dec.out[l])))


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "two-call"])
@pytest.mark.parametrize("name", ["tiny", "c8k"])
def test_step_small_configs_every_row(prism_lib, name, fused):
    P = prism_lib
    cfg = workload.config(name)
    layers = list(workload.generate(cfg, DEV))
    dec = _decoder(P, cfg, fused)
    kqs, scs = {}, {}
    for lay in layers:
        if cfg.is_proposal(lay.index):
            kqs[lay.index], scs[lay.index] = _prefill_kq(P, dec, cfg, lay)
    dec.step([x.q for x in layers], [x.k for x in layers], [x.v for x in layers], kqs, scs)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    for lay in layers:
        l = lay.index
        src = l - l % cfg.group
        _invariants(dec, cfg, l)
        _check_layer(dec, cfg, l, lay, kqs[src], scs[src], _all_rows(cfg))


@pytest.mark.parametrize("name", ["c8k", "c32k_b4", "c128k", "ragged16"])
def test_step_full_size_sampled(prism_lib, name):
    """First proposal group's first two layers at the full sizes."""
    P = prism_lib
    cfg = workload.config(name)
    want = [0, 1]
    layers = list(workload.generate(cfg, DEV, layers=want))
    cfg2 = cfg.replace(num_layers=2)
    dec = _decoder(P, cfg2)
    kqs, scs = {}, {}
    kqs[0], scs[0] = _prefill_kq(P, dec, cfg, layers[0])
    dec.step([x.q for x in layers], [x.k for x in layers], [x.v for x in layers], kqs, scs)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    rng = np.random.default_rng(11)
    rows = sorted({(int(rng.integers(cfg.batch)), int(rng.integers(cfg.num_kv_heads))) for _ in range(3)}
                  | {(cfg.batch - 1, cfg.num_kv_heads - 1)})
    for lay in layers:
        _invariants(dec, cfg2, lay.index)
        _check_layer(dec, cfg2, lay.index, lay, kqs[0], scs[0], rows)
    del layers, dec
    torch.cuda.empty_cache()


def test_step_int2_keys_c8k_every_row(prism_lib):
    """A whole c8k step with INT2 proposal keys: pools against the INT2
    oracle, then refine and attention as in the int8 path."""
    P = prism_lib
    cfg = workload.config("c8k")
    layers = list(workload.generate(cfg, DEV))
    dec = PrismDecoder(cfg.seqlens, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, P.BF16,
                       cfg.num_layers, cfg.group, cfg.kappa_p, cfg.kappa, device=DEV, keys="int2")
    codes, params = {}, {}
    for lay in layers:
        if cfg.is_proposal(lay.index):
            H, T, D = lay.k.shape
            codes[lay.index] = torch.zeros((H, T, D // 4), dtype=torch.uint8, device=DEV)
            params[lay.index] = torch.zeros((H, T, D // 32, 2), dtype=torch.int16, device=DEV)
            P.quantize_k_int2(dec.p, lay.k, codes[lay.index], params[lay.index])
    dec.step([x.q for x in layers], [x.k for x in layers], [x.v for x in layers], codes, params)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    cu = cfg.cu_seqlens
    rows = _all_rows(cfg)
    for lay in layers:
        l = lay.index
        _invariants(dec, cfg, l)
        src = l - l % cfg.group
        if l == src:
            opool, ocnt, osc = pipeline.propose_layer_int2(lay.q, codes[l].cpu().numpy(),
                                                           params[l].cpu().numpy().view(np.uint16), cu,
                                                           cfg.kappa_p, rows=rows)
            gpool, gpc = _np(dec.pool[src]), _np(dec.pool_cnt[src])
            for (b, h) in rows:
                n = int(ocnt[b, h])
                assert int(gpc[b, h]) == n
                check_index_set(gpool[b, h, :n], opool[b, h, :n], lambda t: osc[(b, h)][t],
                                f"L{l} int2 pool {b},{h}")
        # refine + attention on the GPU's own pool (cascade control)
        gpool, gpc = _np(dec.pool[src]), _np(dec.pool_cnt[src])
        gidx, gcnt = _np(dec.idx[l]), _np(dec.cnt[l])
        oidx, ocnt, orr = pipeline.refine_layer(lay.q, lay.k, cu, gpool, gpc, cfg.kappa, rows=rows)
        for (b, h) in rows:
            n = int(gpc[b, h])
            r = dict(zip(gpool[b, h, :n].tolist(), orr[(b, h)].tolist()))
            c = int(ocnt[b, h])
            check_index_set(gidx[b, h, :c], oidx[b, h, :c], lambda t: r[t], f"L{l} idx {b},{h}")
        oout, _ = pipeline.attend_layer(lay.q, lay.k, lay.v, cu, gidx, gcnt, dec.scale, rows=rows)
        assert np.abs(_np(dec.out[l]) - oout).max() <= atol_for(cfg.dtype)


def test_decode_loop_grows_one_sequence(prism_lib):
    """A decode loop over one growing sequence: the cache holds spare rows,
    one step graph is captured once, and before each replay the sequence
    grows by one token, whose K/V rows every layer appends (the proposal
    layer's scorer quantizes its key row).  After every step the proposal
    codes match the oracle's quantizer bit for bit, and pools, index sets
    and outputs match the oracle at that length (c8k shapes, four layers)."""
    P = prism_lib
    steps = 3
    cfg = workload.config("c8k").replace(num_layers=4)
    layers = list(workload.generate(cfg, DEV))
    cap = cfg.seqlens[0]
    L0 = cap - steps
    # the rows the loop appends: kept aside, then overwritten in the cache
    news = [(lay.k[:, L0:].clone(), lay.v[:, L0:].clone()) for lay in layers]
    for lay in layers:
        lay.k[:, L0:] = 7.0
        lay.v[:, L0:] = -7.0
    dec = PrismDecoder([L0], cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, P.BF16,
                       cfg.num_layers, cfg.group, cfg.kappa_p, cfg.kappa, device=DEV, capacity=cap)
    assert dec.scorer_appends
    kqs, scs = {}, {}
    for lay in layers:
        if cfg.is_proposal(lay.index):
            kqs[lay.index], scs[lay.index] = _prefill_kq(P, dec, cfg, lay)
    qbuf = [lay.q.clone() for lay in layers]
    knbuf = [torch.empty((1, cfg.num_kv_heads, cfg.head_dim), dtype=torch.bfloat16, device=DEV)
             for _ in layers]
    vnbuf = [torch.empty_like(x) for x in knbuf]
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        dec.lengths_to_device()
        dec.step(qbuf, [x.k for x in layers], [x.v for x in layers], kqs, scs, k_new=knbuf,
                 v_new=vnbuf)
    gen = torch.Generator(device="cpu").manual_seed(77)
    for t in range(steps):
        dec.grow(1)
        L = L0 + t + 1
        for l, lay in enumerate(layers):
            qbuf[l].copy_((lay.q.float().cpu() + 0.3 * torch.randn(lay.q.shape, generator=gen))
                          .to(torch.bfloat16))
            knbuf[l].copy_(news[l][0][:, t][None])
            vnbuf[l].copy_(news[l][1][:, t][None])
        g.replay()
        torch.cuda.synchronize()
        assert dec.device_status() == 0
        assert int(dec.p.cu_dev[-1]) == L
        cfg_t = cfg.replace(seqlens=(L,))
        for l, lay in enumerate(layers):
            # the cache as the step left it: rows < L with this step's token at L - 1
            assert torch.equal(lay.k[:, L - 1], news[l][0][:, t])
            assert torch.equal(lay.v[:, L - 1], news[l][1][:, t])
            view = workload.Layer(l, qbuf[l], lay.k[:, :L], lay.v[:, :L])
            if cfg.is_proposal(l):
                okq, osc = pipeline.quantize_layer(view.k)
                assert np.array_equal(_np(kqs[l][:, :L]), okq)
                assert np.array_equal(_np(scs[l][:, :L]).view(np.uint32), osc.view(np.uint32))
            src = l - l % cfg.group
            _invariants(dec, cfg_t, l)
            _check_layer(dec, cfg_t, l, view, kqs[src][:, :L], scs[src][:, :L], _all_rows(cfg_t))
    del g


def test_step_group_sum_c8k_every_row(prism_lib):
    """A whole c8k step with the group-sum selection variant (the proposal
    scorer and the refined layers sum the group's query heads): every row of
    every layer against the oracle's sum mode.  The step appends the token's
    rows (the sum variant rides on the scorer that quantizes them)."""
    P = prism_lib
    cfg = workload.config("c8k")
    layers = list(workload.generate(cfg, DEV))
    dec = _decoder(P, cfg, group_agg="sum")
    kqs, scs = {}, {}
    for lay in layers:
        if cfg.is_proposal(lay.index):
            kqs[lay.index], scs[lay.index] = _prefill_kq(P, dec, cfg, lay)
    # this token's rows: the cache already holds them at L - 1 (generated), so
    # appending them again leaves the cache as the oracle sees it
    L = cfg.seqlens[0]
    k_new = [lay.k[:, L - 1][None].clone() for lay in layers]
    v_new = [lay.v[:, L - 1][None].clone() for lay in layers]
    dec.step([x.q for x in layers], [x.k for x in layers], [x.v for x in layers], kqs, scs,
             k_new=k_new, v_new=v_new)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    for lay in layers:
        l = lay.index
        src = l - l % cfg.group
        _invariants(dec, cfg, l)
        _check_layer(dec, cfg, l, lay, kqs[src], scs[src], _all_rows(cfg), agg="sum")


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("name", ["c8k", "tiny"])
def test_step_softmax_mass_every_row(prism_lib, name, fused):
    """A whole step with the softmax-mass selection (the refined layers rank
    pool members by the group's attention mass: fused in prism_refine_decode,
    or prism_refine_mass then the sparse decode; the proposal layers keep the
    maximum): every row of every layer against the oracle's mass mode, sets
    up to near-ties of the mass, outputs within the tolerance."""
    P = prism_lib
    cfg = workload.config(name)
    layers = list(workload.generate(cfg, DEV))
    dec = _decoder(P, cfg, fused=fused, group_agg="mass")
    assert dec.fused == fused
    kqs, scs = {}, {}
    for lay in layers:
        if cfg.is_proposal(lay.index):
            kqs[lay.index], scs[lay.index] = _prefill_kq(P, dec, cfg, lay)
    dec.step([x.q for x in layers], [x.k for x in layers], [x.v for x in layers], kqs, scs)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    for lay in layers:
        l = lay.index
        src = l - l % cfg.group
        _invariants(dec, cfg, l)
        _check_layer(dec, cfg, l, lay, kqs[src], scs[src], _all_rows(cfg), agg="mass")


def _spoil_last_rows(layers, cu, kqs, scs):
    """Overwrite every sequence's last cache row (K, V, and the proposal codes
    and scales) so that only the step's own appends can restore them."""
    for lay in layers:
        for b in range(len(cu) - 1):
            if cu[b + 1] > cu[b]:
                lay.k[:, cu[b + 1] - 1] = 7.0
                lay.v[:, cu[b + 1] - 1] = -7.0
                if lay.index in kqs:
                    kqs[lay.index][:, cu[b + 1] - 1] = 99
                    scs[lay.index][:, cu[b + 1] - 1] = 5.0


@pytest.mark.parametrize("name", ["c128k", "ragged16", "c32k_b4"])
def test_step_timed_sequence_full_size_every_row(prism_lib, name):
    """The call sequence the benchmark times, at full size, on every row of a
    whole proposal group: the token's K/V rows are handed in (k_new/v_new),
    so the proposal layer's scorer quantizes the new key rows itself
    (prism_propose_append) and every refined layer appends its rows inside
    the fused kernel; consecutive refined layers overlap through programmatic
    dependent launch; the step is one captured CUDA graph, replayed twice.
    Before each replay the cache's last rows (K, V, codes, scales) are
    spoiled, so the checks see only what the replay itself wrote.  Every
    (sequence, KV head) row of every layer is then compared with the
    oracle: codes bit for bit, pools and index sets exactly up to near-ties,
    outputs within the bf16 tolerance."""
    P = prism_lib
    full = workload.config(name)
    cfg = full.replace(num_layers=full.group)
    layers = list(workload.generate(cfg, DEV))
    cu = cfg.cu_seqlens
    nz = [b for b in range(cfg.batch) if cu[b + 1] > cu[b]]
    saved = [({b: lay.k[:, cu[b + 1] - 1].clone() for b in nz},
              {b: lay.v[:, cu[b + 1] - 1].clone() for b in nz}) for lay in layers]
    # this token's rows, [B][Hkv][d] per layer, as bench.py builds them
    rows = torch.tensor([cu[b + 1] - 1 for b in nz], dtype=torch.long, device=DEV)
    k_new = [lay.k[:, rows].transpose(0, 1).contiguous() for lay in layers]
    v_new = [lay.v[:, rows].transpose(0, 1).contiguous() for lay in layers]
    dec = PrismDecoder(cfg.seqlens, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, P.BF16,
                       cfg.num_layers, cfg.group, cfg.kappa_p, cfg.kappa, device=DEV,
                       capacity=cfg.total_tokens)
    assert dec.scorer_appends
    kqs, scs = {}, {}
    for lay in layers:
        if cfg.is_proposal(lay.index):
            kqs[lay.index], scs[lay.index] = _prefill_kq(P, dec, cfg, lay)
    qs, ks, vs = [x.q for x in layers], [x.k for x in layers], [x.v for x in layers]
    s = torch.cuda.Stream()

    def step():
        dec.step(qs, ks, vs, kqs, scs, quantize_new=True, k_new=k_new, v_new=v_new)

    with torch.cuda.stream(s):
        _spoil_last_rows(layers, cu, kqs, scs)
        step()  # eager once, as the benchmark does before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    for rep in range(2):
        for x in dec.idx + dec.out:
            x.fill_(-3)
        for lp in dec.pool:
            dec.pool[lp].fill_(-3)
        _spoil_last_rows(layers, cu, kqs, scs)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        assert dec.device_status() == 0
    # the appends: the cache's last rows are this token's rows again
    for lay, (kl, vl) in zip(layers, saved):
        for b in nz:
            assert torch.equal(lay.k[:, cu[b + 1] - 1], kl[b]), (lay.index, b)
            assert torch.equal(lay.v[:, cu[b + 1] - 1], vl[b]), (lay.index, b)
    every = _all_rows(cfg)
    okq = {}
    for lay in layers:
        l = lay.index
        if cfg.is_proposal(l):
            okq[l] = pipeline.quantize_layer(lay.k)
            assert np.array_equal(_np(kqs[l]), okq[l][0]), f"L{l} codes"
            assert np.array_equal(_np(scs[l]).view(np.uint32), okq[l][1].view(np.uint32)), f"L{l} scales"
    for lay in layers:
        l = lay.index
        src = l - l % cfg.group
        _invariants(dec, cfg, l)
        _check_layer(dec, cfg, l, lay, okq[src][0], okq[src][1], every)
    del g, layers, dec
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["c8k", "ragged16"])
def test_step_quantized_proposal_selection_every_row(prism_lib, name):
    """The other reading of what a proposal layer attends over: its own set
    is the top kappa of its pool by the proposal scores (prism_propose_topk,
    no exact rescoring), and its attention runs over that set; the refined
    layers are unchanged.  Every row of a proposal group against the oracle
    in that mode (ragged16: the first group, four layers), with the token's
    rows handed in as the benchmark does."""
    P = prism_lib
    full = workload.config(name)
    cfg = full.replace(num_layers=full.group)
    layers = list(workload.generate(cfg, DEV))
    cu = cfg.cu_seqlens
    nz = [b for b in range(cfg.batch) if cu[b + 1] > cu[b]]
    rows = torch.tensor([cu[b + 1] - 1 for b in nz], dtype=torch.long, device=DEV)
    k_new = [lay.k[:, rows].transpose(0, 1).contiguous() for lay in layers]
    v_new = [lay.v[:, rows].transpose(0, 1).contiguous() for lay in layers]
    dec = PrismDecoder(cfg.seqlens, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, P.BF16,
                       cfg.num_layers, cfg.group, cfg.kappa_p, cfg.kappa, device=DEV,
                       proposal_select="quantized")
    kqs, scs = {}, {}
    for lay in layers:
        if cfg.is_proposal(lay.index):
            kqs[lay.index], scs[lay.index] = _prefill_kq(P, dec, cfg, lay)
    dec.step([x.q for x in layers], [x.k for x in layers], [x.v for x in layers], kqs, scs,
             k_new=k_new, v_new=v_new)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    every = _all_rows(cfg)
    lay0 = layers[0]
    okq, osc = pipeline.quantize_layer(lay0.k)
    opool, ocnt, oscore = pipeline.propose_layer(lay0.q, okq, osc, cu, cfg.kappa_p)
    gpool, gpc = _np(dec.pool[0]), _np(dec.pool_cnt[0])
    for (b, h) in every:
        n = int(ocnt[b, h])
        assert int(gpc[b, h]) == n
        check_index_set(gpool[b, h, :n], opool[b, h, :n], lambda t: oscore[(b, h)][t], f"pool {b},{h}")
    # the proposal layer's own set on the GPU's pool, from the oracle's scores
    oidx, ocnt2 = pipeline.pool_topk_layer(oscore, gpool, gpc, cfg.kappa)
    gidx, gcnt = _np(dec.idx[0]), _np(dec.cnt[0])
    for (b, h) in every:
        c = int(ocnt2[b, h])
        assert int(gcnt[b, h]) == c
        check_index_set(gidx[b, h, :c], oidx[b, h, :c], lambda t: oscore[(b, h)][t], f"L0 idx {b},{h}")
        assert set(gidx[b, h, :c].tolist()) <= set(gpool[b, h, :int(gpc[b, h])].tolist())
    oout, olse = pipeline.attend_layer(lay0.q, lay0.k, lay0.v, cu, gidx, gcnt, dec.scale)
    tol = atol_for(cfg.dtype)
    assert np.abs(_np(dec.out[0]) - oout).max() <= tol
    assert np.abs(_np(dec.lse[0]) - olse).max() <= 10 * tol
    # the refined layers as in the default mode
    for lay in layers[1:]:
        _invariants(dec, cfg, lay.index)
        _check_layer(dec, cfg, lay.index, lay, okq, osc, every)


@pytest.mark.parametrize("sets", ["q_head", "sequence"])
@pytest.mark.parametrize("name", ["c8k", "ragged16"])
def test_step_selection_granularity_every_row(prism_lib, name, sets):
    """The selection-granularity variants over a whole proposal group, every
    row: one set per query head over the group's pool, or one pool and one
    set per sequence shared by every head.  Pools against the oracle (its
    proposal scores in that granularity), sets on the GPU's own pools, and
    attention on the GPU's own sets (cascade control)."""
    P = prism_lib
    full = workload.config(name)
    cfg = full.replace(num_layers=full.group)
    layers = list(workload.generate(cfg, DEV))
    cu = cfg.cu_seqlens
    dec = PrismDecoder(cfg.seqlens, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, P.BF16,
                       cfg.num_layers, cfg.group, cfg.kappa_p, cfg.kappa, device=DEV, sets=sets)
    kqs, scs = {}, {}
    for lay in layers:
        if cfg.is_proposal(lay.index):
            kqs[lay.index], scs[lay.index] = _prefill_kq(P, dec, cfg, lay)
    dec.step([x.q for x in layers], [x.k for x in layers], [x.v for x in layers], kqs, scs)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    lay0 = layers[0]
    okq, osc = pipeline.quantize_layer(lay0.k)
    gpool, gpc = _np(dec.pool[0]), _np(dec.pool_cnt[0])
    tol = atol_for(cfg.dtype)
    if sets == "sequence":
        opool, ocnt, oscore = pipeline.propose_layer_seq(lay0.q, okq, osc, cu, cfg.kappa_p)
        for b in range(cfg.batch):
            n = int(ocnt[b])
            assert int(gpc[b, 0]) == n
            check_index_set(gpool[b, 0, :n], opool[b, :n], lambda t: oscore[b][t], f"seq pool {b}")
    else:
        opool, ocnt, oscore = pipeline.propose_layer(lay0.q, okq, osc, cu, cfg.kappa_p)
        for (b, h) in _all_rows(cfg):
            n = int(ocnt[b, h])
            assert int(gpc[b, h]) == n
            check_index_set(gpool[b, h, :n], opool[b, h, :n], lambda t: oscore[(b, h)][t], f"pool {b},{h}")
    for lay in layers:
        l = lay.index
        gidx, gcnt = _np(dec.idx[l]), _np(dec.cnt[l])
        if sets == "sequence":
            oidx, ocnt2, orr = pipeline.refine_layer_seq(lay.q, lay.k, cu, gpool[:, 0], gpc[:, 0], cfg.kappa)
            for b in range(cfg.batch):
                n, c = int(gpc[b, 0]), int(ocnt2[b])
                assert int(gcnt[b, 0]) == c
                r = dict(zip(gpool[b, 0, :n].tolist(), orr[b].tolist()))
                check_index_set(gidx[b, 0, :c], oidx[b, :c], lambda t: r[t], f"L{l} seq idx {b}")
                assert set(gidx[b, 0, :c].tolist()) <= set(gpool[b, 0, :n].tolist())
            oout, olse = pipeline.attend_layer_sets(lay.q, lay.k, lay.v, cu, gidx[:, 0], gcnt[:, 0],
                                                    "sequence", dec.scale)
        else:
            oidx, ocnt2, orr = pipeline.refine_layer_heads(lay.q, lay.k, cu, gpool, gpc, cfg.kappa)
            G = cfg.G
            for b in range(cfg.batch):
                for hq in range(cfg.num_q_heads):
                    h = hq // G
                    n, c = int(gpc[b, h]), int(ocnt2[b, hq])
                    assert int(gcnt[b, hq]) == c
                    r = dict(zip(gpool[b, h, :n].tolist(), orr[(b, hq)].tolist()))
                    check_index_set(gidx[b, hq, :c], oidx[b, hq, :c], lambda t: r[t], f"L{l} idx {b},{hq}")
                    assert set(gidx[b, hq, :c].tolist()) <= set(gpool[b, h, :n].tolist())
            oout, olse = pipeline.attend_layer_sets(lay.q, lay.k, lay.v, cu, gidx, gcnt, "q_head",
                                                    dec.scale)
        assert np.abs(_np(dec.out[l]) - oout).max() <= tol, l
        assert np.abs(_np(dec.lse[l]) - olse).max() <= 10 * tol, l


@pytest.mark.parametrize("name", ["c8k", "ragged16"])
def test_step_host_matches_device_step(prism_lib, name):
    """PrismDecoder.step_host (the token's rows from page-locked host memory,
    the outputs back to it, one copy per proposal group each way on a side
    stream) in one captured graph gives bit for bit the outputs of the
    device-resident step on the same inputs, over two groups; replayed
    twice."""
    P = prism_lib
    full = workload.config(name)
    cfg = full.replace(num_layers=full.group * 2)
    layers = list(workload.generate(cfg, DEV))
    cu = cfg.cu_seqlens
    nz = [b for b in range(cfg.batch) if cu[b + 1] > cu[b]]
    rows = torch.tensor([cu[b + 1] - 1 for b in nz], dtype=torch.long, device=DEV)
    k_new = torch.stack([lay.k[:, rows].transpose(0, 1).contiguous() for lay in layers])
    v_new = torch.stack([lay.v[:, rows].transpose(0, 1).contiguous() for lay in layers])
    q_all = torch.stack([lay.q for lay in layers])
    ks, vs = [x.k for x in layers], [x.v for x in layers]
    dec = PrismDecoder(cfg.seqlens, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, P.BF16,
                       cfg.num_layers, cfg.group, cfg.kappa_p, cfg.kappa, device=DEV,
                       capacity=cfg.total_tokens)
    kqs, scs = {}, {}
    for lay in layers:
        if cfg.is_proposal(lay.index):
            kqs[lay.index], scs[lay.index] = _prefill_kq(P, dec, cfg, lay)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dec.step([q_all[l] for l in range(cfg.num_layers)], ks, vs, kqs, scs, quantize_new=True,
                 k_new=k_new, v_new=v_new)
    torch.cuda.synchronize()
    ref = dec.out_all.clone()
    io = dec.host_io()
    for l in range(cfg.num_layers):
        io.q_host[l].copy_(q_all[l])
        io.k_new_host[l].copy_(k_new[l])
        io.v_new_host[l].copy_(v_new[l])
    cs = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        dec.step_host(io, ks, vs, kqs, scs, cs)
    for rep in range(2):
        io.out_host.fill_(55.0)
        dec.out_all.fill_(-3.0)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        assert dec.device_status() == 0
        bad = [l for l in range(cfg.num_layers) if not torch.equal(io.out_host[l], ref[l].cpu())]
        dev_bad = [l for l in range(cfg.num_layers) if not torch.equal(dec.out_all[l], ref[l])]
        assert not bad, (rep, bad, dev_bad)
    del g, layers, dec
    torch.cuda.empty_cache()

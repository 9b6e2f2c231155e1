"""One decode step of Prism Attention over every layer, through the C ABI.

Layer schedule (Prism Attention, sec. 5.3 "Accuracy-efficiency trade-off":
in the "g x" setting one layer in every x is a proposal layer; the pages
inherit the partition from an offline calibration, sec. 4 Overview, which is
replaced here by the periodic map ``layer % group == 0``):

  proposal layer l:  the token's key rows are quantized into the proposal
                     codes and the codes are scored (prism_propose_append,
                     or prism_quantize_k then prism_propose / their INT2
                     forms) -> candidate pool of kappa_p positions;
  every layer l:     prism_refine_decode on the latest pool: exact rescoring,
                     top kappa, sparse flash-decode and merge in one launch,
                     appending the layer's new K/V rows -> out[l], lse[l]
                     (or prism_refine then prism_sparse_decode).

A proposal layer also refines its own pool and attends over the refined set
(every layer attends over kappa exactly rescored tokens).  All buffers are
allocated once by torch; a step only enqueues library calls on one stream,
so it can be captured in a CUDA graph.  A decode loop over one growing
sequence (grow / advance_on_device) replays one captured step per token.
"""
from __future__ import annotations

import contextlib
import math
from typing import List, Optional

import torch

from . import prism


class PrismDecoder:
    def __init__(self, seqlens, num_q_heads: int, num_kv_heads: int, head_dim: int, dtype: int,
                 num_layers: int, group: int, kappa_p: int, kappa: int, device="cuda",
                 softmax_scale: Optional[float] = None, fused: bool = True, keys: str = "int8",
                 capacity: Optional[int] = None, group_agg: str = "max",
                 proposal_select: str = "exact", sets: str = "kv_head"):
        self.dev = torch.device(device)
        self.p = prism.Problem(seqlens, num_q_heads, num_kv_heads, head_dim, dtype, device=self.dev,
                               capacity=capacity)
        self.B, self.Hq, self.Hkv, self.D = len(seqlens), num_q_heads, num_kv_heads, head_dim
        self.num_layers, self.group = num_layers, group
        self.kappa_p, self.kappa = kappa_p, kappa
        self.scale = float(torch.tensor(1.0 / math.sqrt(head_dim), dtype=torch.float32)) \
            if softmax_scale is None else float(softmax_scale)
        B, Hkv, Hq, D = self.B, self.Hkv, self.Hq, self.D
        i32 = dict(dtype=torch.int32, device=self.dev)
        f32 = dict(dtype=torch.float32, device=self.dev)
        self.proposal_layers = [l for l in range(num_layers) if l % group == 0]
        # selection granularity: one pool and set per (sequence, KV head)
        # ("kv_head", the default reading); a set per query head over the
        # group's pool ("q_head"); one pool and set per sequence shared by
        # every head ("sequence").  The last two run the two-call path.
        assert sets in ("kv_head", "q_head", "sequence")
        self.sets = sets
        self.sets_code = {"kv_head": prism.SETS_KV_HEAD, "q_head": prism.SETS_Q_HEAD,
                          "sequence": prism.SETS_SEQUENCE}[sets]
        if sets != "kv_head":
            fused = False
        ph = 1 if sets == "sequence" else Hkv       # pool rows per sequence
        sh = {"kv_head": Hkv, "q_head": Hq, "sequence": 1}[sets]  # set rows per sequence
        self.pool = {l: torch.full((B, ph, kappa_p), -1, **i32) for l in self.proposal_layers}
        self.pool_cnt = {l: torch.zeros((B, ph), **i32) for l in self.proposal_layers}
        self.idx = [torch.full((B, sh, kappa), -1, **i32) for _ in range(num_layers)]
        self.cnt = [torch.zeros((B, sh), **i32) for _ in range(num_layers)]
        # per-layer outputs are views of one buffer (one device-to-host copy)
        self.out_all = torch.zeros((num_layers, B, Hq, D), **f32)
        self.lse_all = torch.zeros((num_layers, B, Hq), **f32)
        self.out = [self.out_all[l] for l in range(num_layers)]
        self.lse = [self.lse_all[l] for l in range(num_layers)]
        # the newly appended token of every sequence (packed row index), with
        # a page-locked host mirror that grow() advances
        last = [c - 1 for c in self.p.cu_host[1:].tolist()]
        rows = torch.tensor([r for r, L in zip(last, seqlens) if L > 0], dtype=torch.int32)
        self._new_rows_host = rows.pin_memory() if self.dev.type == "cuda" else rows.clone()
        self.new_rows = rows.to(self.dev)

        def ws(op, kp=0, k=0):
            n = prism.workspace_size(self.p, op, kp, k)
            return torch.zeros(n, dtype=torch.uint8, device=self.dev)

        self.ws_q = ws(prism.OP_QUANTIZE)
        self.ws_prop = ws(prism.OP_PROPOSE, kappa_p)
        self.ws_ref = ws(prism.OP_REFINE, kappa_p, kappa)
        self.ws_dec = ws(prism.OP_SPARSE_DECODE, 0, kappa)
        self.ws_rd = ws(prism.OP_REFINE_DECODE, kappa_p, kappa)
        self.ws_dense = None
        # refined layers in one fused call (refine -> select -> sparse decode)
        self.fused = fused
        # proposal keys: "int8" (kq int8 [Hkv][T][d], k_scale fp32 [Hkv][T]) or
        # "int2" (codes uint8 [Hkv][T][d/4], params int16 [Hkv][T][d/32][2])
        assert keys in ("int8", "int2")
        self.keys = keys
        # int8 proposal layers of a fused step hand the new key rows to the
        # scorer (prism_propose_append), which quantizes them itself; the
        # fused refined layer after it appends the rows to the cache
        self.scorer_appends = (fused and keys == "int8" and dtype == prism.BF16 and head_dim == 128
                               and num_q_heads // num_kv_heads <= 8)
        # how the G query heads of a KV head combine into its selection
        # score: "max" (the default reading), "sum" (the variant, carried by
        # the scorer that takes the new rows and by the fused refined layer)
        # or "mass" (refined selections only, fused or prism_refine_mass in
        # the two-call path: the proposal layers keep the max)
        assert group_agg in ("max", "sum", "mass")
        self.mass = group_agg == "mass"
        if sets != "kv_head" and (keys != "int8" or group_agg != "max"):
            raise ValueError("the q_head / sequence granularities take int8 keys and the maximum")
        if group_agg == "sum" and not self.scorer_appends:
            raise ValueError("group_agg='sum' needs the fused step with int8 keys (bf16, d = 128, G <= 8)")
        self.sum_group = group_agg == "sum"
        # what a proposal layer attends over: "exact" (it refines its own pool
        # like every layer, the default reading) or "quantized" (the top kappa
        # of its pool by the proposal scores it just computed, no rescoring)
        assert proposal_select in ("exact", "quantized")
        self.proposal_select = proposal_select

    def workspaces(self) -> List[torch.Tensor]:
        return [w for w in (self.ws_q, self.ws_prop, self.ws_ref, self.ws_dec, self.ws_rd,
                            self.ws_dense) if w is not None]

    def layer(self, l: int, q, k, v, kq=None, k_scale=None, quantize_new: bool = True,
              k_new=None, v_new=None, k_next=None, overlap: bool = False, stream=None):
        """Enqueue one layer of the step (kq/k_scale -- or INT2 codes/params --
        required at proposal layers).

        k_new / v_new ([B][Hkv][d]), when given, are first written to the last
        position of every sequence (the token being decoded).  overlap: the
        previous kernel on the stream is the fused refined layer before this
        one, so this layer's launch may begin before it ends."""
        p = self.p
        proposal = l % self.group == 0
        # the scorer quantizes the new key rows itself (int8 keys, fused step)
        scorer_new = proposal and self.scorer_appends and k_new is not None and quantize_new
        # a fused refined layer appends the new rows itself
        fused_append = self.fused and k_new is not None and (not proposal or scorer_new)
        if k_new is not None and not fused_append:
            prism.append_kv(p, k_new, v_new, k, v, stream=stream)
        if scorer_new:
            prism.propose_append(p, q, k_new, kq, k_scale, self.kappa_p, self.pool[l], self.pool_cnt[l],
                                 self.ws_prop, sum_group=self.sum_group, stream=stream)
        elif proposal:
            if self.sum_group:
                raise ValueError("group_agg='sum' proposals need this token's key rows (k_new)")
            if self.keys == "int2":
                if quantize_new and self.new_rows.numel():
                    prism.quantize_k_int2(p, k, kq, k_scale, tok_rows=self.new_rows, ws=self.ws_q,
                                          stream=stream)
                prism.propose_int2(p, q, kq, k_scale, self.kappa_p, self.pool[l], self.pool_cnt[l],
                                   self.ws_prop, stream=stream)
            else:
                if quantize_new and self.new_rows.numel():
                    prism.quantize_k(p, k, kq, k_scale, tok_rows=self.new_rows, ws=self.ws_q,
                                     stream=stream)
                prism.propose_ex(p, q, kq, k_scale, self.kappa_p, self.pool[l], self.pool_cnt[l],
                                 self.sets_code, self.ws_prop, stream=stream)
        src = l - l % self.group
        if proposal and self.proposal_select == "quantized":
            prism.propose_topk(p, self.ws_prop, self.pool[l], self.pool_cnt[l], self.kappa_p, self.kappa,
                               self.idx[l], self.cnt[l], self.ws_ref, stream=stream)
            if fused_append:  # no refined-layer call appends this layer's rows
                prism.append_kv(p, k_new, v_new, k, v, stream=stream)
            prism.sparse_decode(p, q, k, v, self.idx[l], self.cnt[l], self.kappa, self.scale,
                                self.out[l], self.ws_dec, lse=self.lse[l], stream=stream)
            return
        if self.fused:
            prism.refine_decode(p, q, k, v, self.pool[src], self.pool_cnt[src], self.kappa_p,
                                self.kappa, self.scale, self.idx[l], self.cnt[l], self.out[l],
                                self.ws_rd, lse=self.lse[l],
                                k_new=k_new if fused_append else None,
                                v_new=v_new if fused_append else None, k_prefetch=k_next,
                                overlap=overlap, sum_group=self.sum_group, mass=self.mass, stream=stream)
            return
        if self.mass:
            prism.refine_mass(p, q, k, self.pool[src], self.pool_cnt[src], self.kappa_p, self.kappa,
                              self.scale, self.idx[l], self.cnt[l], self.ws_ref, stream=stream)
        else:
            prism.refine_ex(p, q, k, self.pool[src], self.pool_cnt[src], self.kappa_p, self.kappa,
                            self.idx[l], self.cnt[l], self.sets_code, self.ws_ref, stream=stream)
        prism.sparse_decode_ex(p, q, k, v, self.idx[l], self.cnt[l], self.kappa, self.scale,
                               self.sets_code, self.out[l], self.ws_dec, lse=self.lse[l], stream=stream)

    def step(self, qs, ks, vs, kqs, scales, quantize_new: bool = True, k_new=None, v_new=None,
             stream=None):
        """One decode step over every layer.  qs/ks/vs (and k_new/v_new) are
        per-layer sequences; kqs/scales are indexed by proposal layer."""
        for l in range(self.num_layers):
            pl = l % self.group == 0
            self.layer(l, qs[l], ks[l], vs[l], kqs[l] if pl else None, scales[l] if pl else None,
                       quantize_new=quantize_new,
                       k_new=None if k_new is None else k_new[l],
                       v_new=None if v_new is None else v_new[l],
                       overlap=self.fused and not pl and l > 0, stream=stream)

    def host_io(self, dtype=torch.bfloat16) -> "HostIO":
        """Page-locked host buffers for step_host, with their device twins."""
        return HostIO(self, dtype)

    def step_host(self, io: "HostIO", ks, vs, kqs, scales, copy_stream, quantize_new: bool = True):
        """One decode step whose token inputs start, and whose outputs end,
        in page-locked host memory: the caller writes this token's rows into
        io.q_host / io.k_new_host / io.v_new_host and reads io.out_host
        after the step.  The copies move a proposal group (`group` layers)
        at a time, one copy per group each way, and meet the layers only at
        group boundaries, where the step has no overlapped launch to lose:
          - every group's rows go up on copy_stream, the first group's first;
            the first layer waits for them, the second group for the rest;
          - each group's outputs go down on copy_stream once its last layer
            ends, while the next group runs.
        The current stream joins copy_stream at the end, so the whole step can
        be captured in one CUDA graph."""
        main = torch.cuda.current_stream()
        L, gsz = self.num_layers, self.group
        copy_stream.wait_stream(main)
        up0, up = torch.cuda.Event(), torch.cuda.Event()
        with torch.cuda.stream(copy_stream):
            io.dev_in[0].copy_(io.host_in[0], non_blocking=True)
            up0.record(copy_stream)
            if io.groups > 1:
                io.dev_in[1:].copy_(io.host_in[1:], non_blocking=True)
                up.record(copy_stream)
        main.wait_event(up0)
        for l in range(L):
            pl = l % gsz == 0
            if l == gsz:
                main.wait_event(up)
            self.layer(l, io.q_dev[l], ks[l], vs[l], kqs[l] if pl else None, scales[l] if pl else None,
                       quantize_new=quantize_new, k_new=io.k_new_dev[l], v_new=io.v_new_dev[l],
                       overlap=self.fused and not pl and l > 0)
            if (l + 1) % gsz == 0 or l + 1 == L:  # the group's outputs go down
                done = torch.cuda.Event()
                done.record(main)
                copy_stream.wait_event(done)
                l0 = l - l % gsz
                with torch.cuda.stream(copy_stream):
                    io.out_host[l0:l + 1].copy_(self.out_all[l0:l + 1], non_blocking=True)
        main.wait_stream(copy_stream)

    def grow(self, n: int = 1):
        """Decode loop over one growing sequence: the last sequence gets n more
        tokens (the next step appends its token at the new last position).
        Host mirrors only; lengths_to_device() sends them, on the stream,
        ahead of the step's kernels (inside a captured step graph, each
        replay copies the mirrors as they are then)."""
        assert self.p.seqlens[-1] > 0, "the last sequence is empty"
        self.p.grow(n)
        self._new_rows_host[-1] += n

    def lengths_to_device(self, stream=None):
        """Enqueue the copies of cu_seqlens and of the new-token rows from
        their host mirrors to the device."""
        ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
        with ctx:
            self.p.cu_dev.copy_(self.p.cu_pin, non_blocking=True)
            self.new_rows.copy_(self._new_rows_host, non_blocking=True)

    def advance_on_device(self, n: int = 1):
        """The device-only form of grow(): the last sequence's length and
        new-token row move on by n on the current stream, so that a captured
        step graph that starts with this call advances the loop on every
        replay without the host (whose mirrors then keep the capture-time
        lengths)."""
        self.p.cu_dev[-1:].add_(n)
        self.new_rows[-1:].add_(n)

    def lengths_from_device(self):
        """Bring the host mirrors back in line with the device lengths (after
        advance_on_device), for calls that size their work from the host
        copy (dense decode)."""
        cu = self.p.cu_dev.cpu()
        self.p.cu_pin.copy_(cu)
        self.p.seqlens = [int(x) for x in (cu[1:] - cu[:-1]).tolist()]
        self._new_rows_host.copy_(self.new_rows.cpu())

    def launches_per_step(self, append: bool) -> int:
        """Kernels one step enqueues (append, quantize, score, select, refine
        score, select, attend, merge)."""
        n = 0
        for l in range(self.num_layers):
            proposal = l % self.group == 0
            scorer_new = proposal and self.scorer_appends and append
            n += 1 if append and ((proposal and not scorer_new) or not self.fused) else 0
            if proposal:
                n += (1 if self.new_rows.numel() and not scorer_new else 0) + 2
            if proposal and self.proposal_select == "quantized":
                n += (1 if append and self.fused and scorer_new else 0) + 2 + 2
                continue
            n += 1 if self.fused else 2 + 2 + (1 if self.mass else 0)
            if self.sets == "sequence":  # the head maxima of the pool scores (and of the proposal's)
                n += 2 if proposal else 1
        return n

    def dense_layer(self, l: int, q, k, v, out, lse=None, stream=None):
        if self.ws_dense is None:
            n = prism.workspace_size(self.p, prism.OP_DENSE_DECODE)
            self.ws_dense = torch.zeros(n, dtype=torch.uint8, device=self.dev)
        prism.dense_decode(self.p, q, k, v, self.scale, out, self.ws_dense, lse=lse, stream=stream)

    def device_status(self) -> int:
        s = 0
        for w in self.workspaces():
            s |= prism.get_device_status(w)
        return s


class HostIO:
    """Host-side inputs and outputs of PrismDecoder.step_host.  Per proposal
    group, one contiguous page-locked block holds its layers' q, then k_new,
    then v_new rows (so one copy moves a group's inputs), mirrored by a
    device block; q_host[l] ([B][Hq][d]), k_new_host[l] / v_new_host[l]
    ([B][Hkv][d]) and their *_dev twins are views into them.  out_host
    ([L][B][Hq][d] fp32, page-locked) receives every layer's output."""

    def __init__(self, dec: PrismDecoder, dtype=torch.bfloat16):
        L, gsz, B, Hq, Hkv, D = dec.num_layers, dec.group, dec.B, dec.Hq, dec.Hkv, dec.D
        es = torch.tensor([], dtype=dtype).element_size()
        nq, nk = B * Hq * D * es, B * Hkv * D * es  # bytes of one layer's q, k_new rows
        self.groups = (L + gsz - 1) // gsz
        blk = gsz * (nq + 2 * nk)
        self.host_in = torch.zeros((self.groups, blk), dtype=torch.uint8).pin_memory()
        self.dev_in = torch.zeros((self.groups, blk), dtype=torch.uint8, device=dec.dev)

        def views(buf):
            q, kn, vn = [], [], []
            for l in range(L):
                gi, j = divmod(l, gsz)
                row = buf[gi]
                q.append(row[j * nq:(j + 1) * nq].view(dtype).view(B, Hq, D))
                o = gsz * nq + j * nk
                kn.append(row[o:o + nk].view(dtype).view(B, Hkv, D))
                o = gsz * (nq + nk) + j * nk
                vn.append(row[o:o + nk].view(dtype).view(B, Hkv, D))
            return q, kn, vn

        self.q_host, self.k_new_host, self.v_new_host = views(self.host_in)
        self.q_dev, self.k_new_dev, self.v_new_dev = views(self.dev_in)
        self.out_host = torch.zeros((L, B, Hq, D), dtype=torch.float32).pin_memory()

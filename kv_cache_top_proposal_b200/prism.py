"""Thin ctypes binding of libprism.so (C ABI in include/prism.h).

Argument marshalling only: every step runs in the library's CUDA kernels.
Tensors are torch tensors on the GPU; the binding passes their data
pointers, sizes and the current CUDA stream, and raises ``PrismError`` for a
non-OK status.  There is no fallback: if the library is missing the import
fails with instructions to build it.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libprism.so")

F32, BF16 = 0, 1
OP_QUANTIZE, OP_PROPOSE, OP_REFINE, OP_SPARSE_DECODE, OP_DENSE_DECODE, OP_REFINE_DECODE = range(6)
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_SCRATCH_LIMIT = range(7)
NOALLOC_SCRATCH_BYTES = 4 << 20
DEV_BAD_INDEX, DEV_TOO_LONG, DEV_TIMEOUT = 0x1, 0x2, 0x4
MAX_SELECT_ROW = 393216
RD_OVERLAP = 0x1
RD_SUM_GROUP = 0x2
RD_MASS = 0x4
SETS_KV_HEAD, SETS_Q_HEAD, SETS_SEQUENCE = 0, 1, 2
PROPOSE_SUM_GROUP = 0x1
WS_HEADER = 256

EXPORTS = ("prism_workspace_size", "prism_append_kv", "prism_quantize_k", "prism_propose",
           "prism_propose_append", "prism_refine",
           "prism_sparse_decode", "prism_refine_decode", "prism_dense_decode",
           "prism_clear_device_status",
           "prism_get_device_status", "prism_status_str", "prism_sparse_decode_noalloc",
           "prism_quantize_k_int2", "prism_propose_int2", "prism_index_overlap",
           "prism_propose_topk", "prism_propose_ex", "prism_refine_ex", "prism_sparse_decode_ex",
           "prism_refine_mass")


class PrismError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.prism_status_str(status).decode()} (status {status})")


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("cu_seqlens_dev", ctypes.c_void_p),
                ("cu_seqlens_host", ctypes.c_void_p), ("total_tokens", ctypes.c_int64)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m kv_cache_top_proposal_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, S, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
    sp = ctypes.POINTER(Shape)
    sig = {
        "prism_workspace_size": [sp, i32, i32, i32, ctypes.POINTER(ctypes.c_size_t)],
        "prism_append_kv": [sp, P, P, P, P, P],
        "prism_quantize_k": [sp, P, P, P, P, i32, P, S, P],
        "prism_propose": [sp, P, P, P, i32, P, P, P, S, P],
        "prism_propose_append": [sp, P, P, P, P, i32, P, P, ctypes.c_uint32, P, S, P],
        "prism_refine": [sp, P, P, P, P, i32, i32, P, P, P, P, S, P],
        "prism_sparse_decode": [sp, P, P, P, P, P, i32, ctypes.c_float, P, P, P, S, P],
        "prism_refine_decode": [sp, P, P, P, P, P, i32, i32, ctypes.c_float, P, P, P, P, P, P, P,
                                ctypes.c_uint32, P, S, P],
        "prism_dense_decode": [sp, P, P, P, ctypes.c_float, P, P, P, S, P],
        "prism_clear_device_status": [P, S, P],
        "prism_get_device_status": [P, S, P, ctypes.POINTER(ctypes.c_int32)],
        "prism_sparse_decode_noalloc": [sp, P, P, P, P, P, i32, ctypes.c_float, P, P, P, P],
        "prism_quantize_k_int2": [sp, P, P, P, P, i32, P, S, P],
        "prism_propose_int2": [sp, P, P, P, i32, P, P, P, S, P],
        "prism_index_overlap": [i32, P, P, i32, P, P, i32, P, P],
        "prism_propose_topk": [sp, P, S, P, P, i32, i32, P, P, P, S, P],
        "prism_propose_ex": [sp, P, P, P, i32, P, P, ctypes.c_uint32, P, S, P],
        "prism_refine_ex": [sp, P, P, P, P, i32, i32, P, P, ctypes.c_uint32, P, S, P],
        "prism_refine_mass": [sp, P, P, P, P, i32, i32, ctypes.c_float, P, P, P, S, P],
        "prism_sparse_decode_ex": [sp, P, P, P, P, P, i32, ctypes.c_float, ctypes.c_uint32, P, P, P, S,
                                   P],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.prism_status_str.argtypes = [ctypes.c_int]
    lib.prism_status_str.restype = ctypes.c_char_p
    return lib


_lib = _load()


def library():
    return _lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, where: str):
    if status != OK:
        raise PrismError(status, where)


class Problem:
    """A layer-shape descriptor (the C ``prism_shape``) plus its cu_seqlens.

    ``seqlens`` are the per-sequence context lengths; the device copy of
    cu_seqlens lives on ``device`` and the host mirror in an array that this
    object keeps alive (page-locked when ``device`` is a GPU, so a captured
    graph can copy it).  ``capacity`` (default: the total length) is the row
    count of every per-token array; rows past the last sequence are spare,
    for a decode loop that grows the last sequence (``grow``).
    """

    def __init__(self, seqlens: Sequence[int], num_q_heads: int, num_kv_heads: int, head_dim: int,
                 dtype: int, device="cuda", cu_dev=None, capacity: Optional[int] = None):
        import torch

        cu = np.zeros(len(seqlens) + 1, np.int32)
        cu[1:] = np.cumsum(np.asarray(seqlens, np.int64)).astype(np.int32)
        host = torch.from_numpy(cu)
        if torch.device(device).type == "cuda":
            host = host.pin_memory()
        self.cu_pin = host                # host mirror (the C shape points at it)
        self.cu_host = host.numpy()       # the same memory, as numpy
        self.cu_dev = cu_dev if cu_dev is not None else host.to(device)
        self.seqlens = [int(x) for x in seqlens]
        self.capacity = int(cu[-1]) if capacity is None else int(capacity)
        if self.capacity < int(cu[-1]):
            raise ValueError("capacity below the total length")
        self.shape = Shape(len(seqlens), num_q_heads, num_kv_heads, head_dim, dtype,
                           ctypes.c_void_p(self.cu_dev.data_ptr()),
                           ctypes.c_void_p(host.data_ptr()), self.capacity)

    @property
    def ref(self):
        return ctypes.byref(self.shape)

    @property
    def total_tokens(self) -> int:
        """Rows of every per-token array (the capacity)."""
        return self.capacity

    def grow(self, n: int = 1):
        """The last sequence gets n more tokens, in the host mirror only; copy
        ``cu_pin`` to ``cu_dev`` on the stream before the kernels that should
        see it (decoder.PrismDecoder.lengths_to_device)."""
        if int(self.cu_host[-1]) + n > self.capacity:
            raise ValueError("the last sequence would outgrow the capacity")
        self.cu_host[-1] += n
        self.seqlens[-1] += n


def workspace_size(p: Problem, op: int, kappa_p: int = 0, kappa: int = 0) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.prism_workspace_size(p.ref, op, kappa_p, kappa, ctypes.byref(n)), "workspace_size")
    return n.value


def _nbytes(ws) -> int:
    return 0 if ws is None else ws.numel() * ws.element_size()


def append_kv(p: Problem, k_new, v_new, k_cache, v_cache, stream=None):
    _check(_lib.prism_append_kv(p.ref, _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                _stream(stream)), "append_kv")


def quantize_k(p: Problem, k, kq, k_scale, tok_rows=None, ws=None, stream=None):
    n = 0 if tok_rows is None else int(tok_rows.numel())
    _check(_lib.prism_quantize_k(p.ref, _ptr(k), _ptr(kq), _ptr(k_scale), _ptr(tok_rows), n,
                                 _ptr(ws), _nbytes(ws), _stream(stream)), "quantize_k")


def propose(p: Problem, q, kq, k_scale, kappa_p: int, pool, pool_cnt, ws, stream=None):
    _check(_lib.prism_propose(p.ref, _ptr(q), _ptr(kq), _ptr(k_scale), kappa_p, _ptr(pool),
                              _ptr(pool_cnt), _ptr(ws), _nbytes(ws), _stream(stream)), "propose")


def propose_append(p: Problem, q, k_new, kq, k_scale, kappa_p: int, pool, pool_cnt, ws,
                   sum_group: bool = False, stream=None):
    """propose with this token's key rows k_new [B][Hkv][d] quantized into kq / k_scale at
    position L_b - 1 by the scorer itself (bf16, d = 128, G <= 8).  sum_group: the
    group's query heads are summed instead of maxed (PRISM_PROPOSE_SUM_GROUP)."""
    _check(_lib.prism_propose_append(p.ref, _ptr(q), _ptr(k_new), _ptr(kq), _ptr(k_scale), kappa_p,
                                     _ptr(pool), _ptr(pool_cnt),
                                     PROPOSE_SUM_GROUP if sum_group else 0, _ptr(ws), _nbytes(ws),
                                     _stream(stream)), "propose_append")


def quantize_k_int2(p: Problem, k, codes, params, tok_rows=None, ws=None, stream=None):
    """INT2 keys: codes [Hkv][T][d/4] uint8, params [Hkv][T][d/32][2] int16/uint16 (fp16 bits of step, zero point)."""
    n = 0 if tok_rows is None else int(tok_rows.numel())
    _check(_lib.prism_quantize_k_int2(p.ref, _ptr(k), _ptr(codes), _ptr(params), _ptr(tok_rows), n,
                                      _ptr(ws), _nbytes(ws), _stream(stream)), "quantize_k_int2")


def propose_int2(p: Problem, q, codes, params, kappa_p: int, pool, pool_cnt, ws, stream=None):
    _check(_lib.prism_propose_int2(p.ref, _ptr(q), _ptr(codes), _ptr(params), kappa_p, _ptr(pool),
                                   _ptr(pool_cnt), _ptr(ws), _nbytes(ws), _stream(stream)),
           "propose_int2")


def refine(p: Problem, q, k, pool, pool_cnt, kappa_p: int, kappa: int, idx, cnt, ws, logits=None,
           stream=None):
    _check(_lib.prism_refine(p.ref, _ptr(q), _ptr(k), _ptr(pool), _ptr(pool_cnt), kappa_p, kappa,
                             _ptr(idx), _ptr(cnt), _ptr(logits), _ptr(ws), _nbytes(ws),
                             _stream(stream)), "refine")


def propose_topk(p: Problem, propose_ws, pool, pool_cnt, kappa_p: int, kappa: int, idx, cnt, ws,
                 stream=None):
    """The proposal layer's own top-kappa from the scores its proposal call
    left in propose_ws (no exact rescoring); ws sized by OP_REFINE."""
    _check(_lib.prism_propose_topk(p.ref, _ptr(propose_ws), _nbytes(propose_ws), _ptr(pool),
                                   _ptr(pool_cnt), kappa_p, kappa, _ptr(idx), _ptr(cnt), _ptr(ws),
                                   _nbytes(ws), _stream(stream)), "propose_topk")


def sparse_decode(p: Problem, q, k, v, idx, cnt, kappa: int, softmax_scale: float, out, ws,
                  lse=None, stream=None):
    _check(_lib.prism_sparse_decode(p.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt), kappa,
                                    float(softmax_scale), _ptr(out), _ptr(lse), _ptr(ws),
                                    _nbytes(ws), _stream(stream)), "sparse_decode")


def refine_decode(p: Problem, q, k, v, pool, pool_cnt, kappa_p: int, kappa: int,
                  softmax_scale: float, idx, cnt, out, ws, lse=None, k_new=None, v_new=None,
                  k_prefetch=None, overlap: bool = False, sum_group: bool = False, mass: bool = False,
                  stream=None):
    """Refined layer in one call; k_new / v_new ([B][Hkv][d]) are appended
    at the last position of every sequence first.  overlap: the launch may
    begin before the previous kernel on the stream ends (see PRISM_RD_OVERLAP);
    sum_group: the exact score sums the group's query heads (PRISM_RD_SUM_GROUP);
    mass: the selection ranks by the group's softmax mass (PRISM_RD_MASS)."""
    _check(_lib.prism_refine_decode(p.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(pool), _ptr(pool_cnt),
                                    kappa_p, kappa, float(softmax_scale), _ptr(idx), _ptr(cnt),
                                    _ptr(out), _ptr(lse), _ptr(k_new), _ptr(v_new),
                                    _ptr(k_prefetch),
                                    (RD_OVERLAP if overlap else 0) | (RD_SUM_GROUP if sum_group else 0)
                                    | (RD_MASS if mass else 0),
                                    _ptr(ws),
                                    _nbytes(ws), _stream(stream)),
           "refine_decode")


def dense_decode(p: Problem, q, k, v, softmax_scale: float, out, ws, lse=None, stream=None):
    _check(_lib.prism_dense_decode(p.ref, _ptr(q), _ptr(k), _ptr(v), float(softmax_scale),
                                   _ptr(out), _ptr(lse), _ptr(ws), _nbytes(ws), _stream(stream)),
           "dense_decode")


def sparse_decode_noalloc(p: Problem, q, k, v, idx, cnt, kappa: int, softmax_scale: float, out,
                          status, lse=None, stream=None):
    """prism_sparse_decode without a workspace, for callers that may not
    allocate device memory at the call: the partials live in the library's
    fixed 4 MiB per-device scratch.  `status` is a device int32 tensor the
    kernels OR bad-index bits into.  Calls that overlap on the GPU race on
    the shared scratch; the first call on a device must precede any stream
    capture."""
    _check(_lib.prism_sparse_decode_noalloc(p.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt),
                                            kappa, float(softmax_scale), _ptr(out), _ptr(lse),
                                            _ptr(status), _stream(stream)),
           "sparse_decode_noalloc")


def clear_device_status(ws, stream=None):
    _check(_lib.prism_clear_device_status(_ptr(ws), _nbytes(ws), _stream(stream)), "clear_status")


def get_device_status(ws, stream=None) -> int:
    c = ctypes.c_int32(0)
    _check(_lib.prism_get_device_status(_ptr(ws), _nbytes(ws), _stream(stream), ctypes.byref(c)),
           "get_device_status")
    return c.value


def index_overlap(a, cnt_a, b, cnt_b, out, stream=None):
    """out[r] = |a[r, :cnt_a[r]] intersect b[r, :cnt_b[r]]| for ascending
    index sets a [rows][stride_a], b [rows][stride_b] (int32, device)."""
    rows = int(cnt_a.numel())
    assert int(cnt_b.numel()) == rows and int(out.numel()) == rows
    _check(_lib.prism_index_overlap(rows, _ptr(a), _ptr(cnt_a), int(a.shape[-1]), _ptr(b),
                                    _ptr(cnt_b), int(b.shape[-1]), _ptr(out), _stream(stream)),
           "index_overlap")


def propose_ex(p: Problem, q, kq, k_scale, kappa_p: int, pool, pool_cnt, sets: int, ws, stream=None):
    """prism_propose at a selection granularity (SETS_*); SETS_SEQUENCE
    writes one pool per sequence, pool [B][kappa_p], pool_cnt [B]."""
    _check(_lib.prism_propose_ex(p.ref, _ptr(q), _ptr(kq), _ptr(k_scale), kappa_p, _ptr(pool),
                                 _ptr(pool_cnt), sets, _ptr(ws), _nbytes(ws), _stream(stream)),
           "propose_ex")


def refine_ex(p: Problem, q, k, pool, pool_cnt, kappa_p: int, kappa: int, idx, cnt, sets: int, ws,
              stream=None):
    """prism_refine at a selection granularity: SETS_Q_HEAD writes idx
    [B][Hq][kappa], SETS_SEQUENCE idx [B][kappa] from pool [B][kappa_p]."""
    _check(_lib.prism_refine_ex(p.ref, _ptr(q), _ptr(k), _ptr(pool), _ptr(pool_cnt), kappa_p, kappa,
                                _ptr(idx), _ptr(cnt), sets, _ptr(ws), _nbytes(ws), _stream(stream)),
           "refine_ex")


def refine_mass(p: Problem, q, k, pool, pool_cnt, kappa_p: int, kappa: int, softmax_scale: float, idx,
                cnt, ws, stream=None):
    """prism_refine_mass: the refined set by the group's softmax mass over the
    pool (workspace of OP_REFINE)."""
    _check(_lib.prism_refine_mass(p.ref, _ptr(q), _ptr(k), _ptr(pool), _ptr(pool_cnt), kappa_p, kappa,
                                  float(softmax_scale), _ptr(idx), _ptr(cnt), _ptr(ws), _nbytes(ws),
                                  _stream(stream)),
           "refine_mass")


def sparse_decode_ex(p: Problem, q, k, v, idx, cnt, kappa: int, softmax_scale: float, sets: int, out,
                     ws, lse=None, stream=None):
    _check(_lib.prism_sparse_decode_ex(p.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt), kappa,
                                       float(softmax_scale), sets, _ptr(out), _ptr(lse), _ptr(ws),
                                       _nbytes(ws), _stream(stream)), "sparse_decode_ex")

"""CPU oracle for the Prism Attention decode hot path (test infrastructure).

The arithmetic lives in ``prism_oracle.c`` (plain sequential C, fp32 for
everything that decides a selection, fp64 for attention outputs); this module
compiles it with gcc and wraps it with ctypes.  ``pipeline`` drives it over
whole layers and decode steps.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import this package.  The CUDA library
never calls it, and it never calls the CUDA library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "prism_oracle.c")
_SO = os.path.join(_HERE, "_build", "libprism_oracle.so")

# No FMA contraction and no fast-math: sums are evaluated exactly as written,
# feature index ascending, each product and each sum rounded to fp32.
CFLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-frounding-math"]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build`` (idempotent)."""
    os.makedirs(os.path.dirname(_SO), exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.oracle_quantize_rows.argtypes = [P, i64, i32, P, P]
        lib.oracle_topk_ascending.argtypes = [P, i32, i32, P]
        lib.oracle_topk_ascending.restype = i32
        lib.oracle_propose_scores.argtypes = [P, i32, i32, P, P, i32, P]
        lib.oracle_propose_row.argtypes = [P, i32, i32, P, P, i32, i32, P, P]
        lib.oracle_propose_row.restype = i32
        lib.oracle_refine_scores.argtypes = [P, i32, i32, P, P, i32, P]
        lib.oracle_refine_row.argtypes = [P, i32, i32, P, P, i32, i32, P, P]
        lib.oracle_refine_row.restype = i32
        lib.oracle_attend.argtypes = [P, i32, P, P, P, i32, f64, P, P]
        lib.oracle_propose_scores_sum.argtypes = [P, i32, i32, P, P, i32, P]
        lib.oracle_propose_row_sum.argtypes = [P, i32, i32, P, P, i32, i32, P, P]
        lib.oracle_propose_row_sum.restype = i32
        lib.oracle_refine_scores_sum.argtypes = [P, i32, i32, P, P, i32, P]
        lib.oracle_refine_row_sum.argtypes = [P, i32, i32, P, P, i32, i32, P, P]
        lib.oracle_refine_row_sum.restype = i32
        lib.oracle_f32_to_f16.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_f16.restype = ctypes.c_uint16
        lib.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f32.restype = ctypes.c_float
        lib.oracle_quantize_int2_rows.argtypes = [P, i64, i32, P, P]
        lib.oracle_propose_scores_int2.argtypes = [P, i32, i32, P, P, i32, P]
        lib.oracle_propose_row_int2.argtypes = [P, i32, i32, P, P, i32, i32, P, P]
        lib.oracle_propose_row_int2.restype = i32
        lib.oracle_set_overlap.argtypes = [P, i32, P, i32]
        lib.oracle_set_overlap.restype = i32
        lib.oracle_pool_topk.argtypes = [P, P, i32, i32, P]
        lib.oracle_pool_topk.restype = i32
        lib.oracle_refine_row_heads.argtypes = [P, i32, i32, P, P, i32, i32, P, P]
        lib.oracle_refine_row_heads.restype = i32
        lib.oracle_propose_row_seq.argtypes = [P, i32, i32, i32, P, P, i32, i32, P, P]
        lib.oracle_propose_row_seq.restype = i32
        lib.oracle_refine_row_seq.argtypes = [P, i32, i32, i32, P, i32, P, i32, i32, P, P]
        lib.oracle_refine_row_seq.restype = i32
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def quantize_rows(k):
    """int8 symmetric per-row quantization -> (kq [rows, d] int8, scale [rows] f32)."""
    k = _f32(k)
    rows, d = k.shape
    kq = np.empty((rows, d), np.int8)
    sc = np.empty((rows,), np.float32)
    _L().oracle_quantize_rows(_p(k), rows, d, _p(kq), _p(sc))
    return kq, sc


def topk_ascending(s, k: int) -> np.ndarray:
    """Top-k indices of s (score desc, lower index wins ties), ascending."""
    s = _f32(s)
    out = np.empty((max(min(k, s.size), 1),), np.int32)
    m = _L().oracle_topk_ascending(_p(s), s.size, k, _p(out))
    return out[:m].copy()


AGGS = ("max", "sum")  # how the G query heads of a KV head combine into one selection score


def _sfx(agg: str) -> str:
    if agg not in AGGS:
        raise ValueError(f"agg must be one of {AGGS}")
    return "" if agg == "max" else "_sum"


def propose_scores(q, kq, scale, agg: str = "max") -> np.ndarray:
    """s_t = scale_t * max_g (or sum_g) sum_j q[g, j] * kq[t, j] (fp32, j ascending)."""
    q, kq, scale = _f32(q), np.ascontiguousarray(kq, dtype=np.int8), _f32(scale)
    G, d = q.shape
    L = kq.shape[0]
    s = np.empty((L,), np.float32)
    getattr(_L(), "oracle_propose_scores" + _sfx(agg))(_p(q), G, d, _p(kq), _p(scale), L, _p(s))
    return s


def propose_row(q, kq, scale, kappa_p: int, agg: str = "max"):
    """(pool ascending int32 [min(kappa_p, L)], proposal scores [L])."""
    q, kq, scale = _f32(q), np.ascontiguousarray(kq, dtype=np.int8), _f32(scale)
    G, d = q.shape
    L = kq.shape[0]
    s = np.empty((max(L, 1),), np.float32)
    pool = np.empty((max(min(kappa_p, L), 1),), np.int32)
    m = getattr(_L(), "oracle_propose_row" + _sfx(agg))(_p(q), G, d, _p(kq), _p(scale), L, kappa_p,
                                                        _p(pool), _p(s))
    return pool[:m].copy(), s[:L].copy()


def pool_topk(scores, pool, kappa: int) -> np.ndarray:
    """The proposal layer's own set under the quantized-selection reading:
    the top min(kappa, |pool|) pool members by their proposal scores
    (scores [L], one per position), positions ascending."""
    s, pool = _f32(scores), _i32(pool)
    idx = np.empty((max(min(kappa, pool.size), 1),), np.int32)
    m = _L().oracle_pool_topk(_p(s), _p(pool), pool.size, kappa, _p(idx))
    return idx[:m].copy()


def refine_scores(q, K, pool, agg: str = "max") -> np.ndarray:
    """r_i = max_g (or sum_g) sum_j q[g, j] * K[pool_i, j] (fp32, j ascending)."""
    q, K, pool = _f32(q), _f32(K), _i32(pool)
    G, d = q.shape
    r = np.empty((max(pool.size, 1),), np.float32)
    getattr(_L(), "oracle_refine_scores" + _sfx(agg))(_p(q), G, d, _p(K), _p(pool), pool.size, _p(r))
    return r[:pool.size].copy()


def refine_row(q, K, pool, kappa: int, agg: str = "max"):
    """(refined positions ascending int32 [min(kappa, |pool|)], exact pool scores)."""
    q, K, pool = _f32(q), _f32(K), _i32(pool)
    G, d = q.shape
    n = pool.size
    r = np.empty((max(n, 1),), np.float32)
    idx = np.empty((max(min(kappa, n), 1),), np.int32)
    m = getattr(_L(), "oracle_refine_row" + _sfx(agg))(_p(q), G, d, _p(K), _p(pool), n, kappa,
                                                       _p(idx), _p(r))
    return idx[:m].copy(), r[:n].copy()


def refine_scores_mass(q, K, pool, softmax_scale: float) -> np.ndarray:
    """Group aggregation by softmax mass (the third reading of how the G query
    heads of a KV head share one set; Prism Attention sec. 4.1 and sec. 6
    leave it open): a pool member's score is the attention mass the group's
    heads put on it, each head's softmax taken over the pool,
        l_g,i = softmax_scale * (q_g . K[pool_i])     the dot product fp32,
                                                      j ascending (the
                                                      one-head exact score)
        r_i   = sum_g exp(l_g,i - max_i' l_g,i') / sum_i' exp(l_g,i' - max_i' l_g,i')
    in fp64 after the dot products, g ascending.  Returns r (fp64)."""
    q, K, pool = _f32(q), _f32(K), _i32(pool)
    G = q.shape[0]
    n = pool.size
    r = np.zeros(n, np.float64)
    if n == 0:
        return r
    for g in range(G):
        dots = refine_scores(q[g:g + 1], K, pool).astype(np.float64)  # exact fp32 dot products
        lg = float(softmax_scale) * dots
        e = np.exp(lg - lg.max())
        r += e / e.sum()
    return r


def refine_row_mass(q, K, pool, kappa: int, softmax_scale: float):
    """(refined positions ascending int32 [min(kappa, |pool|)], masses fp64):
    the top min(kappa, |pool|) members by softmax mass, ties to the lower
    pool slot (the lower position, as the pool is ascending)."""
    pool = _i32(pool)
    r = refine_scores_mass(q, K, pool, softmax_scale)
    order = sorted(range(pool.size), key=lambda i: (-r[i], i))
    take = sorted(order[:min(kappa, pool.size)])
    return pool[np.array(take, np.int64)].astype(np.int32) if take else np.zeros(0, np.int32), r


def attend(q, K, V, idx, softmax_scale: float):
    """fp64 softmax attention of one query head over rows idx (None = all rows)."""
    q, K, V = _f32(q), _f32(K), _f32(V)
    d = q.shape[0]
    if idx is None:
        n, ip = K.shape[0], None
    else:
        idx = _i32(idx)
        n, ip = idx.size, _p(idx)
    out = np.empty((d,), np.float32)
    lse = np.empty((1,), np.float32)
    _L().oracle_attend(_p(q), d, _p(K), _p(V), ip, n, float(softmax_scale), _p(out), _p(lse))
    return out, float(lse[0])


# ---- INT2 proposal keys -----------------------------------------------------

def f32_to_f16_bits(x: float) -> int:
    """fp16 bits of x, round to nearest even."""
    return int(_L().oracle_f32_to_f16(float(np.float32(x))))


def f16_bits_to_f32(h: int) -> float:
    return float(_L().oracle_f16_to_f32(int(h)))


def quantize_int2_rows(k):
    """INT2 per-group quantization -> (codes [rows, d/4] uint8 packed, params
    [rows, d/32, 2] uint16 fp16 bits of (step S, zero point L))."""
    k = _f32(k)
    rows, d = k.shape
    codes = np.empty((rows, d // 4), np.uint8)
    params = np.empty((rows, d // 32, 2), np.uint16)
    _L().oracle_quantize_int2_rows(_p(k), rows, d, _p(codes), _p(params))
    return codes, params


def unpack_int2(codes, d: int) -> np.ndarray:
    """Packed codes [rows, d/4] -> code values [rows, d] (feature f at bits 2 (f mod 4) of byte f / 4)."""
    codes = np.asarray(codes, np.uint8)
    shifts = (2 * (np.arange(d) % 4)).astype(np.uint8)
    return (codes[:, np.arange(d) // 4] >> shifts) & 3


def propose_scores_int2(q, codes, params) -> np.ndarray:
    """s_t = max_g sum over groups of (S * D + L * Q) (fp32, see the C source)."""
    q = _f32(q)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    params = np.ascontiguousarray(params, dtype=np.uint16)
    G, d = q.shape
    L = codes.shape[0]
    s = np.empty((max(L, 1),), np.float32)
    _L().oracle_propose_scores_int2(_p(q), G, d, _p(codes), _p(params), L, _p(s))
    return s[:L].copy()


def propose_row_int2(q, codes, params, kappa_p: int):
    """(pool ascending int32 [min(kappa_p, L)], INT2 proposal scores [L])."""
    q = _f32(q)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    params = np.ascontiguousarray(params, dtype=np.uint16)
    G, d = q.shape
    L = codes.shape[0]
    s = np.empty((max(L, 1),), np.float32)
    pool = np.empty((max(min(kappa_p, L), 1),), np.int32)
    m = _L().oracle_propose_row_int2(_p(q), G, d, _p(codes), _p(params), L, kappa_p, _p(pool), _p(s))
    return pool[:m].copy(), s[:L].copy()


# ---- index overlap (sec. 3 "Observations", Figure 1) -------------------------

def set_overlap(a, b) -> int:
    """|a intersect b| of two strictly ascending index sets."""
    a, b = _i32(a), _i32(b)
    return int(_L().oracle_set_overlap(_p(a), a.size, _p(b), b.size))


# ---- selection granularity variants ------------------------------------------

def refine_row_heads(q, K, pool, kappa: int):
    """Per-query-head sets over a shared pool: (idx [G][min(kappa, n)]
    positions ascending per head, exact scores [G][n])."""
    q, K, pool = _f32(q), _f32(K), _i32(pool)
    G, d = q.shape
    n = pool.size
    idx = np.empty((G, max(kappa, 1)), np.int32)
    r = np.empty((G, max(n, 1)), np.float32)
    m = _L().oracle_refine_row_heads(_p(q), G, d, _p(K), _p(pool), n, kappa, _p(idx), _p(r))
    return idx[:, :m].copy(), r[:, :n].copy()


def propose_row_seq(q, kq, scale, kappa_p: int):
    """One pool per sequence shared by every head: q [Hq][d], kq [Hkv][L][d],
    scale [Hkv][L] -> (pool ascending, head-max proposal scores [L])."""
    q = _f32(q)
    kq = np.ascontiguousarray(kq, dtype=np.int8)
    scale = _f32(scale)
    Hkv, L, d = kq.shape
    G = q.shape[0] // Hkv
    s = np.empty((max(L, 1),), np.float32)
    pool = np.empty((max(min(kappa_p, L), 1),), np.int32)
    m = _L().oracle_propose_row_seq(_p(q), Hkv, G, d, _p(kq), _p(scale), L, kappa_p, _p(pool), _p(s))
    return pool[:m].copy(), s[:L].copy()


def refine_row_seq(q, K, pool, kappa: int):
    """One set per sequence: q [Hq][d], K [Hkv][L][d] -> (positions ascending,
    head-max exact scores of the pool)."""
    q, K, pool = _f32(q), _f32(K), _i32(pool)
    Hkv, L, d = K.shape
    G = q.shape[0] // Hkv
    n = pool.size
    r = np.empty((max(n, 1),), np.float32)
    idx = np.empty((max(min(kappa, n), 1),), np.int32)
    m = _L().oracle_refine_row_seq(_p(q), Hkv, G, d, _p(K), L, _p(pool), n, kappa, _p(idx), _p(r))
    return idx[:m].copy(), r[:n].copy()

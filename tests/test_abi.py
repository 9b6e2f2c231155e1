"""The C-ABI library: it loads, exports every declared entry point, and
rejects bad host-checkable arguments before touching the GPU (these tests
run without a device: validation never dereferences device pointers)."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # a non-null "device pointer" that validation never reads


def _declared():
    src = open(os.path.join(ROOT, "include", "prism.h")).read()
    return re.findall(r"PRISM_API\s+[\w\s\*]+?\b(prism_\w+)\s*\(", src)


def test_exports_every_declared_symbol(prism_lib):
    names = _declared()
    assert len(names) >= 9
    lib = prism_lib.library()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(prism_lib.EXPORTS)


def _shape(prism, seqlens, hq=32, hkv=8, d=128, dtype=1):
    cu = np.zeros(len(seqlens) + 1, np.int32)
    cu[1:] = np.cumsum(seqlens)
    s = prism.Shape(len(seqlens), hq, hkv, d, dtype, ctypes.c_void_p(FAKE),
                    ctypes.c_void_p(cu.ctypes.data), int(cu[-1]))
    return s, cu


def _ws(prism, s, op, kp=0, k=0):
    n = ctypes.c_size_t(0)
    st = prism.library().prism_workspace_size(ctypes.byref(s), op, kp, k, ctypes.byref(n))
    return st, n.value


def test_workspace_sizes(prism_lib):
    P = prism_lib
    s, cu = _shape(P, [1000, 3000])
    st, n = _ws(P, s, P.OP_PROPOSE, 256)
    assert st == P.OK and n >= 256 + 8 * 4000 * 4 and n % 256 == 0
    st, n = _ws(P, s, P.OP_REFINE, 256, 64)
    assert st == P.OK and n >= 256 + 2 * 8 * 256 * 4 * (1 + 4)
    st, n0 = _ws(P, s, P.OP_QUANTIZE)
    assert st == P.OK and n0 == 256
    st, n = _ws(P, s, P.OP_SPARSE_DECODE, 0, 64)
    assert st == P.OK and n > 256
    st, n = _ws(P, s, P.OP_DENSE_DECODE)
    assert st == P.OK and n > 256


@pytest.mark.parametrize("bad", [
    dict(hq=30, hkv=8), dict(hq=4, hkv=8), dict(d=96), dict(dtype=7), dict(hq=8 * 17, hkv=8),
])
def test_bad_shapes_rejected(prism_lib, bad):
    P = prism_lib
    kw = dict(hq=32, hkv=8, d=128, dtype=1)
    kw.update(bad)
    s, cu = _shape(P, [100], **kw)
    st, _ = _ws(P, s, P.OP_PROPOSE, 16)
    assert st in (P.ERR_INVALID_ARG, P.ERR_UNSUPPORTED)


def test_bad_cu_seqlens_rejected(prism_lib):
    P = prism_lib
    s, cu = _shape(P, [100, 50])
    cu[1] = 200  # not monotone
    assert _ws(P, s, P.OP_PROPOSE, 16)[0] == P.ERR_INVALID_ARG
    s, cu = _shape(P, [100, 50])
    s.total_tokens = 149  # fewer rows than cu[B]
    assert _ws(P, s, P.OP_PROPOSE, 16)[0] == P.ERR_INVALID_ARG
    s, cu = _shape(P, [100, 50])
    s.total_tokens = 151  # one spare row past cu[B]: accepted
    assert _ws(P, s, P.OP_PROPOSE, 16)[0] == P.OK
    s, cu = _shape(P, [100])
    cu[0] = 1
    assert _ws(P, s, P.OP_PROPOSE, 16)[0] == P.ERR_INVALID_ARG


def test_calls_validate_before_launch(prism_lib):
    P = prism_lib
    lib = P.library()
    s, cu = _shape(P, [4096])
    ref = ctypes.byref(s)
    f = ctypes.c_void_p(FAKE)
    _, nprop = _ws(P, s, P.OP_PROPOSE, 1024)
    ws = ctypes.c_void_p(FAKE)  # 256-aligned fake workspace
    # null pointers
    assert lib.prism_propose(ref, None, f, f, 1024, f, f, ws, nprop, None) == P.ERR_INVALID_ARG
    # kappa_p < 1
    assert lib.prism_propose(ref, f, f, f, 0, f, f, ws, nprop, None) == P.ERR_INVALID_ARG
    # workspace too small / misaligned
    assert lib.prism_propose(ref, f, f, f, 1024, f, f, ws, nprop - 1, None) == P.ERR_WORKSPACE
    assert lib.prism_propose(ref, f, f, f, 1024, f, f, ctypes.c_void_p(FAKE + 4), nprop,
                             None) == P.ERR_WORKSPACE
    # kappa > kappa_p
    _, nref = _ws(P, s, P.OP_REFINE, 256, 64)
    assert lib.prism_refine(ref, f, f, f, f, 256, 512, f, f, None, ws, nref, None) == P.ERR_INVALID_ARG
    assert lib.prism_refine(ref, f, f, f, f, 256, 0, f, f, None, ws, nref, None) == P.ERR_INVALID_ARG
    # softmax-mass selection: the same bounds, and a finite positive scale
    rm = lib.prism_refine_mass
    assert rm(ref, f, f, f, f, 256, 512, 0.1, f, f, ws, nref, None) == P.ERR_INVALID_ARG
    assert rm(ref, f, f, f, f, 256, 64, 0.0, f, f, ws, nref, None) == P.ERR_INVALID_ARG
    assert rm(ref, f, f, f, f, 256, 64, float("inf"), f, f, ws, nref, None) == P.ERR_INVALID_ARG
    assert rm(ref, None, f, f, f, 256, 64, 0.1, f, f, ws, nref, None) == P.ERR_INVALID_ARG
    assert rm(ref, f, f, f, f, 256, 64, 0.1, f, f, ws, nref - 1, None) == P.ERR_WORKSPACE
    # non-finite softmax scale
    _, ndec = _ws(P, s, P.OP_SPARSE_DECODE, 0, 64)
    assert lib.prism_sparse_decode(ref, f, f, f, f, f, 64, float("nan"), f, None, ws, ndec,
                                   None) == P.ERR_INVALID_ARG
    assert lib.prism_dense_decode(ref, f, f, None, 0.1, f, None, ws, 1 << 30, None) == P.ERR_INVALID_ARG
    assert lib.prism_quantize_k(ref, f, None, f, None, 0, None, 0, None) == P.ERR_INVALID_ARG
    assert lib.prism_get_device_status(None, 0, None, None) == P.ERR_WORKSPACE
    # fused refined layer: unknown flags, a lone new row, misaligned rows
    _, nrd = _ws(P, s, P.OP_REFINE_DECODE, 1024, 256)
    rd = lib.prism_refine_decode
    assert rd(ref, f, f, f, f, f, 1024, 256, 0.1, f, f, f, None, None, None, None, 8, ws, nrd,
              None) == P.ERR_INVALID_ARG
    assert rd(ref, f, f, f, f, f, 1024, 256, 0.1, f, f, f, None, f, None, None, 0, ws, nrd,
              None) == P.ERR_INVALID_ARG
    bad = ctypes.c_void_p(FAKE + 8)
    assert rd(ref, bad, f, f, f, f, 1024, 256, 0.1, f, f, f, None, None, None, None, 0, ws, nrd,
              None) == P.ERR_INVALID_ARG
    assert rd(ref, f, f, f, f, f, 1024, 2048, 0.1, f, f, f, None, None, None, None, 0, ws, nrd,
              None) == P.ERR_INVALID_ARG
    # the softmax-mass flag: not with the group sum, and a positive scale
    assert rd(ref, f, f, f, f, f, 1024, 256, 0.1, f, f, f, None, None, None, None, 2 | 4, ws, nrd,
              None) == P.ERR_INVALID_ARG
    assert rd(ref, f, f, f, f, f, 1024, 256, -0.1, f, f, f, None, None, None, None, 4, ws, nrd,
              None) == P.ERR_INVALID_ARG
    # proposal with the new key rows: unknown flags, missing rows, unsupported head dim
    pa = lib.prism_propose_append
    assert pa(ref, f, f, f, f, 1024, f, f, 2, ws, nprop, None) == P.ERR_INVALID_ARG
    assert pa(ref, f, None, f, f, 1024, f, f, 0, ws, nprop, None) == P.ERR_INVALID_ARG
    s64, cu64 = _shape(P, [100], d=64)  # cu64 stays alive: s64 points at it
    _, n64 = _ws(P, s64, P.OP_PROPOSE, 1024)
    assert pa(ctypes.byref(s64), f, f, f, f, 1024, f, f, 0, ws, n64, None) == P.ERR_UNSUPPORTED


def test_too_long_rows_unsupported(prism_lib):
    P = prism_lib
    s, cu = _shape(P, [P.MAX_SELECT_ROW + 1])
    _, n = _ws(P, s, P.OP_PROPOSE, 1024)
    f = ctypes.c_void_p(FAKE)
    assert P.library().prism_propose(ctypes.byref(s), f, f, f, 1024, f, f, f, n, None) == P.ERR_UNSUPPORTED


def test_status_strings(prism_lib):
    lib = prism_lib.library()
    for code in range(6):
        assert lib.prism_status_str(code)
    assert b"workspace" in lib.prism_status_str(prism_lib.ERR_WORKSPACE)


def test_propose_topk_and_overlap_reject_bad_arguments(prism_lib):
    """Host checks of prism_propose_topk (the proposal workspace and the
    refine workspace are both sized and aligned) and prism_index_overlap."""
    P = prism_lib
    lib = P.library()
    s, cu = _shape(P, [1000, 3000])
    _, nprop = _ws(P, s, P.OP_PROPOSE, 256)
    _, nref = _ws(P, s, P.OP_REFINE, 256, 64)
    f = ctypes.c_void_p(FAKE)

    def call(pws, pn, ws, n, kp=256, k=64):
        return lib.prism_propose_topk(ctypes.byref(s), pws, pn, f, f, kp, k, f, f, ws, n, None)

    assert call(f, nprop - 1, f, nref) == P.ERR_WORKSPACE           # proposal workspace too small
    assert call(f, nprop, f, nref - 1) == P.ERR_WORKSPACE           # refine workspace too small
    assert call(ctypes.c_void_p(FAKE + 16), nprop, f, nref) == P.ERR_WORKSPACE  # misaligned
    assert call(f, nprop, f, nref, kp=64, k=256) == P.ERR_INVALID_ARG  # kappa > kappa_p
    assert call(None, nprop, f, nref) == P.ERR_WORKSPACE
    ov = lib.prism_index_overlap
    assert ov(4, f, f, 0, f, f, 8, f, None) == P.ERR_INVALID_ARG     # stride 0
    assert ov(-1, f, f, 8, f, f, 8, f, None) == P.ERR_INVALID_ARG
    assert ov(4, None, f, 8, f, f, 8, f, None) == P.ERR_INVALID_ARG
    assert ov(0, None, None, 8, None, None, 8, None, None) == P.OK  # nothing to do


def _dense_splits(P, seqlens, hq=32, hkv=8, d=128, dtype=1):
    """Split count of the dense plan, read back from its workspace size:
    a 256-byte header, then partial o [B][Hq][splits][d] and (m, l)
    [B][Hq][splits][2] fp32, each padded to 256 bytes."""
    s, _ = _shape(P, seqlens, hq, hkv, d, dtype)
    st, n = _ws(P, s, P.OP_DENSE_DECODE)
    assert st == P.OK
    per_split = len(seqlens) * hq * (d + 2) * 4
    splits = (n - 256) // per_split
    assert 0 <= (n - 256) - splits * per_split < 512  # the two paddings
    return splits


def test_dense_split_plan(prism_lib):
    """The tensor-core dense kernel runs one CTA per SM (148 planned): equal
    lengths fill one wave of whole 128-row stages; a ragged batch gets
    shorter splits than one wave would give its longest row, so the long rows
    spread over several SMs; fp32 caches keep the staged kernel's two CTAs
    per SM."""
    P = prism_lib
    # c128k: 8 rows, one wave -> floor(148 / 8) = 18 splits of 7296 positions
    assert _dense_splits(P, [131072]) == 18
    # four equal rows of 32768 (32 rows): ceil(32768 / splits) rounded to 128
    sp = _dense_splits(P, [32768] * 4)
    assert 4 <= sp <= 37
    # ragged: a long row among short ones is cut into more pieces than the
    # one-wave plan (148 // 128 = 1 split) would give it
    rng = np.random.default_rng(5)
    ragged = [int(x) for x in rng.integers(4096, 65537, 16)]
    assert _dense_splits(P, ragged) > 1
    # fp32: two CTAs per SM over 8 rows -> ceil(296 / 8) = 37 splits
    assert _dense_splits(P, [131072], dtype=0) == 37

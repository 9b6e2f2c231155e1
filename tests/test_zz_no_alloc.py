"""prism_sparse_decode_noalloc, the sparse decode for callers that may not
allocate device memory at the call, against prism_sparse_decode.

Two calls in a row on different problems (different lengths, heads, index
sets and split plans), each checked against the workspace entry point on the
same inputs: the second call must not see what the first left in the shared
scratch.  The file is collected last and builds its own inputs, so it passes
alone in a fresh process as well as after the other tests.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

DEV = "cuda"


def _inputs(seqlens, hq, hkv, d, dtype, kap, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    T = int(sum(seqlens))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = torch.randn((len(seqlens), hq, d), generator=g).to(tdt).to(DEV)
    k = torch.randn((hkv, T, d), generator=g).to(tdt).to(DEV)
    v = torch.randn((hkv, T, d), generator=g).to(tdt).to(DEV)
    rng = np.random.default_rng(seed)
    B = len(seqlens)
    idx = np.full((B, hkv, kap), -1, np.int32)
    cnt = np.zeros((B, hkv), np.int32)
    for b, L in enumerate(seqlens):
        for h in range(hkv):
            n = min(kap, L) if (b + h) % 3 else min(kap, L) // 2
            idx[b, h, :n] = np.sort(rng.choice(L, n, replace=False))
            cnt[b, h] = n
    return q, k, v, torch.tensor(idx, device=DEV), torch.tensor(cnt, device=DEV)


CASES = [
    # (seqlens, Hq, Hkv, d, dtype, kappa): the full-size decode row first,
    # then a ragged batch with an empty sequence and fewer splits
    ([131072], 32, 8, 128, "bf16", 2048),
    ([5000, 1031, 0, 300], 8, 2, 128, "bf16", 700),
]


def _both(P, prob, q, k, v, idx, cnt, kap, scale, B, hq, d):
    """(workspace status, out, lse) of prism_sparse_decode and (status_dev,
    out, lse) of the no-allocation entry point on the same inputs."""
    ws = torch.zeros(P.workspace_size(prob, P.OP_SPARSE_DECODE, 0, kap), dtype=torch.uint8,
                     device=DEV)
    ref_out = torch.full((B, hq, d), 77.0, device=DEV)
    ref_lse = torch.full((B, hq), 77.0, device=DEV)
    P.sparse_decode(prob, q, k, v, idx, cnt, kap, scale, ref_out, ws, lse=ref_lse)
    out = torch.full((B, hq, d), -55.0, device=DEV)
    lse = torch.full((B, hq), -55.0, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    P.sparse_decode_noalloc(prob, q, k, v, idx, cnt, kap, scale, out, status, lse=lse)
    torch.cuda.synchronize()
    return (P.get_device_status(ws), ref_out, ref_lse), (int(status.item()), out, lse)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice(prism_lib):
    """Same kernels, same split plan and summation order as the workspace
    entry point, so the results must be identical, bit for bit."""
    P = prism_lib
    for i, (seqlens, hq, hkv, d, dtype, kap) in enumerate(CASES):
        prob = P.Problem(seqlens, hq, hkv, d, P.BF16 if dtype == "bf16" else P.F32, device=DEV)
        q, k, v, idx, cnt = _inputs(seqlens, hq, hkv, d, dtype, kap, seed=40 + i)
        scale = float(np.float32(1 / math.sqrt(d)))
        (ws_st, ref_out, ref_lse), (st, out, lse) = _both(P, prob, q, k, v, idx, cnt, kap, scale,
                                                          len(seqlens), hq, d)
        assert ws_st == 0 and st == 0, i
        assert torch.equal(out, ref_out), i
        assert torch.equal(lse, ref_lse), i


@pytest.mark.gpu
def test_noalloc_reports_bad_indices_in_status_dev(prism_lib):
    """An index past its sequence and a count above kappa: the kernels skip
    the bad index and clamp the count without touching memory outside the
    arrays, and the no-allocation call reports both in the caller's status
    word exactly as the workspace entry point reports them in its header."""
    P = prism_lib
    seqlens, hq, hkv, d, kap = [3000, 1200], 8, 2, 128, 256
    prob = P.Problem(seqlens, hq, hkv, d, P.BF16, device=DEV)
    q, k, v, idx, cnt = _inputs(seqlens, hq, hkv, d, "bf16", kap, seed=9)
    idx[0, 1, 5] = seqlens[0]       # one position at L: skipped
    cnt[1, 0] = kap + 7             # one count above kappa: clamped to kappa
    idx[1, 0, :] = torch.arange(kap, dtype=torch.int32, device=DEV)
    scale = float(np.float32(1 / math.sqrt(d)))
    (ws_st, ref_out, ref_lse), (st, out, lse) = _both(P, prob, q, k, v, idx, cnt, kap, scale,
                                                      len(seqlens), hq, d)
    assert ws_st == P.DEV_BAD_INDEX
    assert st == P.DEV_BAD_INDEX
    assert torch.equal(out, ref_out)
    assert torch.equal(lse, ref_lse)


def test_noalloc_rejects_requests_beyond_the_scratch(prism_lib):
    """Host-side check: 4096 sequences x 32 query heads need 68 MB of
    partials, more than the 4 MiB scratch; nothing is enqueued and no device
    pointer is read (so this runs without a GPU)."""
    P = prism_lib
    fake = ctypes.c_void_p(0x10000)
    seqlens = [64] * 4096
    cu = np.zeros(len(seqlens) + 1, np.int32)
    cu[1:] = np.cumsum(seqlens)
    s = P.Shape(len(seqlens), 32, 8, 128, P.BF16, fake, ctypes.c_void_p(cu.ctypes.data), int(cu[-1]))
    st = P.library().prism_sparse_decode_noalloc(ctypes.byref(s), fake, fake, fake, fake, fake, 64,
                                                 0.088, fake, None, fake, None)
    assert st == P.ERR_SCRATCH_LIMIT
    assert b"fixed scratch" in P.library().prism_status_str(st)
    st = P.library().prism_sparse_decode_noalloc(ctypes.byref(s), fake, fake, fake, fake, fake, 64,
                                                 0.088, fake, None, None, None)
    assert st == P.ERR_INVALID_ARG

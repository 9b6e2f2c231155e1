"""Helpers shared by the GPU parity tests (comparison rules only).

Index sets are compared element by element; the only allowed differences
are members whose oracle fp32 score lies within 1e-5 relative of the
oracle's k-th score (the GPU sums in another order, so near-ties may swap).
"""
import numpy as np

REL_TIE = 1e-5
ATOL_BF16 = 2e-3
ATOL_F32 = 1e-5


def check_index_set(got, want, score_of, label=""):
    """got/want: ascending int arrays; score_of(position) -> oracle fp32 score."""
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.size == want.size, f"{label}: count {got.size} != {want.size}"
    if got.size == 0:
        return 0
    assert np.all(np.diff(got) > 0), f"{label}: not strictly ascending"
    if np.array_equal(got, want):
        return 0
    sk = min(score_of(int(t)) for t in want)  # the oracle's k-th score
    tol = REL_TIE * max(abs(sk), 1e-30)
    diff = set(got.tolist()) ^ set(want.tolist())
    for t in diff:
        s = score_of(int(t))
        assert abs(s - sk) <= tol, f"{label}: member {t} score {s} vs k-th {sk} (tol {tol})"
    return len(diff)


def atol_for(dtype_name):
    return ATOL_BF16 if dtype_name == "bf16" else ATOL_F32

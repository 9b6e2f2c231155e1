"""Host-side logic of the decode loop (no GPU): spare rows, growth of the
last sequence and its bounds, the device-only advance, and the sum-variant
guard.  Buffers live on the CPU here; the library is only asked for sizes."""
import numpy as np
import pytest
import torch

from kv_cache_top_proposal_b200 import prism
from kv_cache_top_proposal_b200.decoder import PrismDecoder


def _dec(**kw):
    args = dict(device="cpu", capacity=1000)
    args.update(kw)
    return PrismDecoder([990], 8, 2, 128, prism.BF16, 4, 2, 256, 64, **args)


def test_problem_capacity_and_grow():
    p = prism.Problem([300, 500], 8, 2, 128, prism.BF16, device="cpu", capacity=805)
    assert p.total_tokens == 805 and p.shape.total_tokens == 805
    assert p.cu_host.tolist() == [0, 300, 800]
    p.grow(5)
    assert p.cu_host.tolist() == [0, 300, 805] and p.seqlens == [300, 505]
    with pytest.raises(ValueError):
        p.grow(1)
    with pytest.raises(ValueError):
        prism.Problem([300, 500], 8, 2, 128, prism.BF16, device="cpu", capacity=799)
    # the library sizes workspaces from the capacity (scores for every row)
    n805 = prism.workspace_size(p, prism.OP_PROPOSE, 128)
    q = prism.Problem([300, 500], 8, 2, 128, prism.BF16, device="cpu")
    assert n805 > prism.workspace_size(q, prism.OP_PROPOSE, 128)


def test_decoder_grow_moves_the_new_row_and_the_lengths():
    dec = _dec()
    assert dec.new_rows.tolist() == [989]
    dec.grow(3)
    assert dec.p.cu_host.tolist() == [0, 993] and dec._new_rows_host.tolist() == [992]
    assert dec.p.cu_dev.tolist() == [0, 993]  # on the CPU the device copy is the host array
    dec.lengths_to_device()
    assert dec.new_rows.tolist() == [992]
    with pytest.raises(ValueError):
        dec.grow(8)  # 993 + 8 > 1000


def test_advance_on_device_then_back_to_the_host():
    dec = _dec()
    cu0 = dec.p.cu_dev.clone()
    dec.p.cu_dev = cu0  # a device copy apart from the host mirror, as on a GPU
    dec.advance_on_device(2)
    assert dec.p.cu_dev.tolist() == [0, 992] and dec.new_rows.tolist() == [991]
    assert dec.p.cu_host.tolist() == [0, 990]  # the host mirror keeps the capture-time length
    dec.lengths_from_device()
    assert dec.p.cu_host.tolist() == [0, 992] and dec.p.seqlens == [992]
    assert dec._new_rows_host.tolist() == [991]


def test_launch_counts_and_variant_guard():
    dec = _dec()
    assert dec.scorer_appends
    # per proposal layer: score + select (no append, no quantize); refine_decode on every layer
    assert dec.launches_per_step(append=True) == 2 * 2 + 4
    assert dec.launches_per_step(append=False) == 2 * 3 + 4
    assert _dec(group_agg="sum").sum_group
    with pytest.raises(ValueError):
        _dec(group_agg="sum", keys="int2")
    with pytest.raises(ValueError):
        PrismDecoder([990], 8, 2, 64, prism.BF16, 4, 2, 256, 64, device="cpu", group_agg="sum")

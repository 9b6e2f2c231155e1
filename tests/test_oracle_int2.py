"""Pins for the oracle's INT2 proposal keys (Prism Attention, sec. 4.2: the key
cache read at proposal layers is compressed to INT2 for candidate scoring;
the scheme -- per 32-feature group, asymmetric 2-bit codes with an fp16 zero
point and step -- is this repository's reading of it).

Each pin checks the oracle against something other than itself: numpy's own
float16 conversion, hand-derived cases, the fp64 dot product with the
dequantized key, exact integer arithmetic and the quantizer's closed-form
bounds.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "int2_cases.json")


def test_f16_conversion_matches_numpy_on_every_half():
    # fp16 -> fp32 on all 65536 bit patterns (NaN payloads compared as NaN)
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([oracle.f16_bits_to_f32(int(b)) for b in bits], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f32_to_f16_rounds_like_numpy():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10,
        (rng.standard_normal(20000) * 1e-5).astype(np.float32),        # subnormal halves
        (rng.uniform(60000, 70000, 2000)).astype(np.float32),           # overflow edge
        np.float32([0.0, -0.0, 65504, 65519.99, 65520, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
                    1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 2.0 ** -14 - 2.0 ** -25]),
    ])
    # exact ties of the 11-bit significand: halfway values round to even
    m = rng.integers(1024, 2048, 2000)
    ties = (m * 2 + 1).astype(np.float32) * np.float32(2.0 ** -12)
    vals = np.concatenate([vals, ties, -ties])
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f32_to_f16_bits(float(v)) for v in vals], np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(vals[i]), hex(got[i]), hex(ref[i])) for i in bad[:5]]


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["quantize"], ids=lambda c: c["cite"][:40])
def test_int2_quantize_hand_cases(case):
    k = np.array(case["k"], np.float32)[None]
    codes, params = oracle.quantize_int2_rows(k)
    assert oracle.unpack_int2(codes, k.shape[1])[0].tolist() == case["codes"]
    assert [oracle.f16_bits_to_f32(int(x)) for x in params[0, :, 0]] == case["step"]
    assert [oracle.f16_bits_to_f32(int(x)) for x in params[0, :, 1]] == case["zero"]


def test_int2_packing_layout():
    # feature f lives at bits 2 (f mod 4) of byte f / 4
    k = np.tile(np.float32([0, 1, 2, 3, 3, 2, 1, 0]), 4)[None]
    codes, _ = oracle.quantize_int2_rows(k)
    assert codes[0, 0] == (0 | 1 << 2 | 2 << 4 | 3 << 6)
    assert codes[0, 1] == (3 | 2 << 2 | 1 << 4 | 0 << 6)


def test_int2_quantize_bounds_random():
    rng = np.random.default_rng(1)
    k = (rng.standard_normal((500, 128)) * rng.uniform(0.01, 50, (500, 1))).astype(np.float32)
    k[7] = 2.5  # a constant row: step 0
    codes, params = oracle.quantize_int2_rows(k)
    c = oracle.unpack_int2(codes, 128).reshape(500, 4, 32).astype(np.float64)
    S = params[..., 0].view(np.float16).astype(np.float64)[..., None]
    Lz = params[..., 1].view(np.float16).astype(np.float64)[..., None]
    x = k.reshape(500, 4, 32).astype(np.float64)
    lo, hi = x.min(-1, keepdims=True), x.max(-1, keepdims=True)
    assert np.all((c >= 0) & (c <= 3))
    # zero point and step are the fp16 roundings of lo and (hi - L) / 3
    assert np.all(np.abs(Lz - lo) <= np.abs(lo) * 2.0 ** -11 + 2.0 ** -25)
    ideal = (hi - Lz) / 3
    assert np.all(np.abs(S - ideal) <= ideal * 2.0 ** -11 + 2.0 ** -25)
    # the smallest element maps to code 0, the largest to code 3 (S > 0)
    ar = np.arange(500)[:, None]
    assert np.all(c[ar, np.arange(4), x.argmin(-1)] == 0)
    pos = S[..., 0] > 0
    assert np.all(c[ar, np.arange(4), x.argmax(-1)][pos] == 3)
    assert np.all(c[~pos] == 0) and not pos[7].any()
    # dequantization error: half a step, plus the zero point's and the
    # step's fp16 rounding carried over three steps
    deq = Lz + S * c
    bound = 0.5 * S + np.abs(Lz - lo) + 3 * np.abs(S - ideal) + 1e-6 * np.abs(x).max()
    assert np.all(np.abs(deq - x) <= bound + 1e-12)


def test_int2_scores_equal_dequantized_dot_product():
    rng = np.random.default_rng(2)
    G, d, L = 4, 128, 300
    q = rng.standard_normal((G, d)).astype(np.float32)
    k = rng.standard_normal((L, d)).astype(np.float32)
    codes, params = oracle.quantize_int2_rows(k)
    s = oracle.propose_scores_int2(q, codes, params)
    c = oracle.unpack_int2(codes, d).reshape(L, 4, 32).astype(np.float64)
    S = params[..., 0].view(np.float16).astype(np.float64)[..., None]
    Lz = params[..., 1].view(np.float16).astype(np.float64)[..., None]
    deq = (Lz + S * c).reshape(L, d)
    ref = (deq @ q.astype(np.float64).T).max(1)
    scale = np.abs(deq) @ np.abs(q.astype(np.float64)).T
    assert np.all(np.abs(s - ref) <= 2e-6 * scale.max(1) + 1e-30)


def test_int2_scores_exact_on_integer_data():
    # groups spanning exactly {z, z+1, z+2, z+3} with integer z: step 1, zero
    # point z, codes k - z, so every term is an exact small integer
    rng = np.random.default_rng(3)
    G, d, L = 3, 64, 50
    z = rng.integers(-20, 20, (L, d // 32, 1))
    k = z + np.tile(np.arange(4), (L, d // 32, 8))
    k = rng.permuted(k, axis=2).reshape(L, d).astype(np.float32)
    q = rng.integers(-5, 6, (G, d)).astype(np.float32)
    codes, params = oracle.quantize_int2_rows(k)
    assert np.all(params[..., 0].view(np.float16) == 1)
    s = oracle.propose_scores_int2(q, codes, params)
    exact = (k.astype(np.int64) @ q.astype(np.int64).T).max(1)
    assert np.array_equal(s, exact.astype(np.float32))


def test_int2_proposal_pool_is_brute_force_top_k():
    rng = np.random.default_rng(4)
    G, d, L, kp = 2, 64, 40, 9
    q = rng.standard_normal((G, d)).astype(np.float32)
    k = rng.standard_normal((L, d)).astype(np.float32)
    k[5] = k[11]  # an exact tie: the lower position must win
    codes, params = oracle.quantize_int2_rows(k)
    pool, s = oracle.propose_row_int2(q, codes, params, kp)
    order = sorted(range(L), key=lambda t: (-float(s[t] + 0.0), t))
    assert pool.tolist() == sorted(order[:kp])
    assert np.array_equal(s, oracle.propose_scores_int2(q, codes, params))

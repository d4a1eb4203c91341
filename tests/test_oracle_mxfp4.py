"""Pins of the oracle's MXFP4 decoding, encoding and bf16 rounding.

Each check compares the oracle with something fixed outside it: the OCP MX
value tables (tests/golden), exact powers of two from the standard library,
hand-packed bytes, and torch's own float32 -> bfloat16 conversion.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from oracle import mxfp4


def golden_e2m1():
    return {int(c): float(v) for c, _, v in read_golden("e2m1_values.txt")}


def test_e2m1_table_matches_ocp():
    g = golden_e2m1()
    assert len(g) == 16
    for c in range(16):
        v = mxfp4.e2m1_value(c)
        assert v == g[c]
        assert math.copysign(1.0, v) == math.copysign(1.0, g[c])   # -0.0 at code 8


def test_e8m0_matches_ocp():
    for b, v in read_golden("e8m0_values.txt"):
        got = mxfp4.e8m0_value(int(b))
        if v == "nan":
            assert math.isnan(got)
        else:
            assert got == float.fromhex(v)


def test_dequantize_exhaustive_codes_by_scales():
    """All 16 codes under all 256 scale bytes against table * 2**(e-127)."""
    g = golden_e2m1()
    codes = np.tile(np.arange(16, dtype=np.uint8), 2)            # 32 = one block
    packed = mxfp4.pack_codes(np.tile(codes, (256, 1)))           # [256, 16]
    scales = np.arange(256, dtype=np.uint8).reshape(256, 1)
    w = mxfp4.dequantize(packed, scales)
    for e in range(256):
        for i in range(32):
            want = g[int(codes[i])] * math.ldexp(1.0, e - 127) if e != 255 else math.nan
            got = w[e, i]
            if e == 255:
                assert math.isnan(got)
            else:
                assert got == want, (e, i)


def test_nibble_order_low_first():
    # byte 0x21: element 0 = code 1 (0.5), element 1 = code 2 (1.0)
    # byte 0xF0: element 2 = code 0 (0.0), element 3 = code 15 (-6.0)
    row = np.zeros((1, 16), dtype=np.uint8)
    row[0, 0] = 0x21
    row[0, 1] = 0xF0
    w = mxfp4.dequantize(row, np.array([[127]], dtype=np.uint8))
    assert list(w[0, :4]) == [0.5, 1.0, 0.0, -6.0]


def test_scale_applies_per_32_elements():
    codes = np.full((1, 64), 2, dtype=np.uint8)                   # all 1.0
    w = mxfp4.dequantize(mxfp4.pack_codes(codes), np.array([[127, 129]], dtype=np.uint8))
    assert np.all(w[0, :32] == 1.0) and np.all(w[0, 32:] == 4.0)


def test_round_trip_every_code_and_scale():
    for e in range(1, 255):
        vals = np.array([mxfp4.e2m1_value(c) * math.ldexp(1.0, e - 127) for c in range(16)])
        back = mxfp4.encode_e2m1(vals, e)
        assert list(back) == list(range(16)), e


def test_encoder_ties_to_even():
    for x, code in read_golden("e2m1_rne_ties.txt"):
        assert int(mxfp4.encode_e2m1(np.array([float(x)]), 127)[0]) == int(code), x


def _torch_bf16(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(7)
    xs = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),   # subnormals
        (rng.standard_normal(2000) * 1e38).astype(np.float32),
        np.array([0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 3.3895e38, 3.4e38,
                  2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135], dtype=np.float32),
    ]).astype(np.float64)
    got = mxfp4.round_bf16(xs)
    want = _torch_bf16(xs)
    assert np.array_equal(got, want) or np.array_equal(np.nan_to_num(got), np.nan_to_num(want))
    assert np.array_equal(np.signbit(got), np.signbit(want))


def test_round_bf16_known_values():
    r = mxfp4.round_bf16(np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -30]))
    assert list(r) == [1.0, 1.0 + 2.0 ** -6, 1.0 + 2.0 ** -7]


def test_bf16_bits_round_trip():
    vals = mxfp4.round_bf16(np.random.default_rng(3).standard_normal(1000))
    assert np.array_equal(mxfp4.from_bf16_bits(mxfp4.bf16_bits(vals)), vals)


def test_dequantize_rejects_bad_scale_shape():
    with pytest.raises(ValueError):
        mxfp4.dequantize(np.zeros((2, 16), np.uint8), np.zeros((2, 2), np.uint8))


# ------------------------------------------------- OCP MX conversion (encoder) --

def test_quantize_scale_is_floor_log2_minus_two():
    w = np.zeros((1, 64))
    w[0, 5] = 6.0           # floor(log2 6) = 2 -> X = 2**0
    w[0, 40] = -0.7         # floor(log2 0.7) = -1 -> X = 2**-3
    c, s = mxfp4.quantize_mxfp4(w)
    assert list(s[0]) == [127, 124]
    assert mxfp4.dequantize(c, s)[0, 5] == 6.0
    assert mxfp4.dequantize(c, s)[0, 40] == -0.75   # 0.7 / 2**-3 = 5.6 -> 6


def test_quantize_value_round_trip_of_mxfp4_matrices():
    """Any MXFP4 matrix's values survive quantisation exactly (the scale may
    change when a block's largest code is below 4, the values may not)."""
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, (16, 64 // 2), dtype=np.uint8)
    scales = rng.integers(110, 140, (16, 64 // 32), dtype=np.uint8)
    v = mxfp4.dequantize(codes, scales)
    c2, s2 = mxfp4.quantize_mxfp4(v)
    assert np.array_equal(mxfp4.dequantize(c2, s2), v)


def test_quantize_error_bound_and_nearest_code():
    """Per block 4X <= amax < 8X; an element within +-6X becomes the nearest
    representable value (brute force over the 16 codes), one beyond
    saturates to +-6X; so |q - w| <= 2X."""
    rng = np.random.default_rng(6)
    w = rng.normal(size=(8, 96)) * np.exp(rng.normal(size=(8, 1)) * 3)
    c, s = mxfp4.quantize_mxfp4(w)
    q = mxfp4.dequantize(c, s)
    for r in range(8):
        for b in range(3):
            X = 2.0 ** (int(s[r, b]) - 127)
            blk, qb = w[r, 32 * b:32 * b + 32], q[r, 32 * b:32 * b + 32]
            assert 4 * X <= np.abs(blk).max() < 8 * X
            assert np.abs(qb - blk).max() <= 2 * X
            inside = np.abs(blk) <= 6 * X
            cands = mxfp4.E2M1_TABLE[None, :] * X
            nearest = np.abs(blk[:, None] - cands).min(axis=1)
            assert np.array_equal(np.abs(qb - blk)[inside], nearest[inside])
            assert np.array_equal(qb[~inside], np.sign(blk[~inside]) * 6 * X)


def test_quantize_zero_block_and_bad_input():
    c, s = mxfp4.quantize_mxfp4(np.zeros((2, 32)))
    assert (s == 0).all() and (mxfp4.dequantize(c, s) == 0).all()
    import pytest
    with pytest.raises(ValueError):
        mxfp4.quantize_mxfp4(np.zeros((1, 33)))
    with pytest.raises(ValueError):
        mxfp4.quantize_mxfp4(np.full((1, 32), np.inf))

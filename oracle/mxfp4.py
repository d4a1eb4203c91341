"""MXFP4 decoding, encoding and bf16 rounding (oracle; test infrastructure).

The pages state that the expert weights are stored as OCP MXFP4 ([P3]
"MiMo-v2.5-Pro-UltraSpeed - infra 架构解读", section "FP4 Expert 量化";
[P4] "mimo-tilert-1000tps-trillion-parameter-inference", section
"第一层：FP4 选择性量化") but do not print the format.  The element and scale
encodings below follow the OCP MX v1.0 definition that those sections name:

* an MX block is 32 elements sharing one scale;
* element = E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; the
  exponent field 0 encodes the subnormal 0.5*m; no inf/NaN encodings;
* scale = E8M0: an unsigned 8-bit exponent, value 2**(e - 127); 0xFF is NaN.

Byte packing is not fixed by the format.  Reading taken here: two elements
per byte, element 2j in the low nibble and element 2j+1 in the high nibble;
scale j covers elements [32j, 32j+32) of the same row.
"""
from __future__ import annotations

import math

import numpy as np


def e2m1_value(code: int) -> float:
    """Real value of one 4-bit E2M1 code, from its bit fields."""
    if not 0 <= code <= 15:
        raise ValueError("E2M1 code out of range")
    sign = -1.0 if (code >> 3) & 1 else 1.0
    exp = (code >> 1) & 3
    man = code & 1
    if exp == 0:                       # subnormal: 0.m x 2**(1 - bias)
        mag = 0.5 * man
    else:                              # normal: 1.m x 2**(exp - bias), bias 1
        mag = (1.0 + 0.5 * man) * 2.0 ** (exp - 1)
    return sign * mag


# 16-entry table built from the bit-field rule above.
E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)


def e8m0_value(e: int) -> float:
    """Real value of an E8M0 scale byte: 2**(e-127), NaN for 0xFF."""
    if not 0 <= e <= 255:
        raise ValueError("E8M0 byte out of range")
    if e == 255:
        return math.nan
    return math.ldexp(1.0, e - 127)


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """[R, K/2] packed bytes -> [R, K] codes (low nibble first)."""
    c = np.asarray(codes, dtype=np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = c & 0x0F
    out[..., 1::2] = c >> 4
    return out


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """[R, K] 4-bit codes -> [R, K/2] bytes (inverse of unpack_codes)."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0x0F) | ((c[..., 1::2] & 0x0F) << 4)


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """MXFP4 row-major matrix -> float64 [R, K].

    codes: [R, K/2] uint8, scales: [R, K/32] uint8.  Every value is
    E2M1(code) * 2**(scale-127), exact in float64.
    """
    el = unpack_codes(codes)
    R, K = el.shape
    if scales.shape != (R, K // 32):
        raise ValueError(f"scale shape {scales.shape} does not match codes {(R, K)}")
    vals = E2M1_TABLE[el]
    s = np.asarray(scales, dtype=np.int64)
    mult = np.where(s == 255, np.nan, np.ldexp(1.0, s - 127))
    return vals * np.repeat(mult, 32, axis=1)


def encode_e2m1(x: np.ndarray, scale_byte: int) -> np.ndarray:
    """Nearest E2M1 code of x / 2**(scale-127), ties to the even mantissa.

    Saturates at +-6.  Signed zeros keep their sign (code 0 or 8).  Used for
    round-trip checks of the decoder; the path itself never encodes.
    """
    v = np.asarray(x, dtype=np.float64) / math.ldexp(1.0, scale_byte - 127)
    mags = E2M1_TABLE[:8]                    # 0, .5, 1, 1.5, 2, 3, 4, 6
    a = np.abs(v)
    d = np.abs(a[..., None] - mags)          # distance to every magnitude
    nearest = d == d.min(axis=-1, keepdims=True)
    even = (np.arange(8) & 1) == 0
    # a unique nearest magnitude wins; of two tied ones, the even code wins
    best = np.where(nearest.sum(axis=-1) > 1,
                    np.argmax(nearest & even, axis=-1),
                    np.argmax(nearest, axis=-1))
    best = np.where(a >= 6.0, 7, best)
    neg = np.signbit(v)
    return (best + 8 * neg).astype(np.uint8)


def quantize_mxfp4(w: np.ndarray):
    """Real matrix [R, K] (K a multiple of 32) -> MXFP4 (codes [R, K/2] uint8,
    scales [R, K/32] uint8), by the OCP MX v1.0 conversion: per 32-element
    block the shared scale is X = 2**(floor(log2(amax)) - 2) (2 = the largest
    E2M1 exponent), clamped to the E8M0 range, and each element becomes the
    nearest E2M1 code of v / X, ties to even, saturating at +-6.  An all-zero
    block takes the smallest scale (byte 0).  This is the format's own
    encoder, for a weight quantiser; the verify path never quantises."""
    w = np.asarray(w, dtype=np.float64)
    R, K = w.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    if not np.isfinite(w).all():
        raise ValueError("non-finite input")
    codes = np.zeros((R, K), dtype=np.uint8)
    scales = np.zeros((R, K // 32), dtype=np.uint8)
    for r in range(R):
        for b in range(K // 32):
            blk = w[r, 32 * b:32 * b + 32]
            amax = float(np.abs(blk).max())
            if amax == 0.0:
                byte = 0
            else:
                _, ex = math.frexp(amax)              # amax = m * 2**ex, m in [0.5, 1)
                byte = min(254, max(0, (ex - 1) - 2 + 127))
            scales[r, b] = byte
            codes[r, 32 * b:32 * b + 32] = encode_e2m1(blk, byte)
    return pack_codes(codes), scales


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), as float64.

    bfloat16 = 1 sign, 8 exponent (bias 127), 7 stored mantissa bits, with
    subnormals; overflow past the largest finite value goes to +-inf.
    """
    a = np.asarray(x, dtype=np.float64)
    out = np.empty_like(a)
    fin = np.isfinite(a)
    v = a[fin]
    _, e = np.frexp(v)                       # v = m * 2**e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                  # below 2**-126 the quantum is fixed
    quantum = np.ldexp(1.0, e - 8)           # 8 significant bits
    r = np.rint(v / quantum) * quantum       # rint: half to even
    big = np.ldexp(255.0 / 128.0, 127)       # largest finite bfloat16
    r = np.where(np.abs(r) > big, np.copysign(np.inf, r), r)
    out[fin] = r
    out[~fin] = a[~fin]
    return out


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Bit patterns (uint16) of values that are exactly bfloat16."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """uint16 bfloat16 bit patterns -> float64 values."""
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)

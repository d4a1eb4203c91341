"""Accuracy of the activation encoding the tensor-core FFN feeds to kind::mxf4.

The kernel writes each bf16 activation row as eight E2M1 terms,
v = sum_t 2**s_t * c_t, where term t is the nearest E2M1 code of what terms
0..t-1 left over, against the scale 2**s_t that puts the row's largest
remaining magnitude in (3, 6].  This test restates that rule with the
oracle's E2M1 encoder on random bf16 rows of the FFN's shapes and checks the
property the design relies on: the eight terms give the row back to a
relative L2 error far below the FFN tolerance, most elements exactly.  It
pins the algorithm, not the CUDA code (the GPU parity tests do that).
"""
import math

import numpy as np

from mxfp4_moe_block_b200 import synth
from oracle import mxfp4


def _scale_exp(amax: float) -> int:
    """s with amax / 2**s in (3, 6]: E2M1's largest magnitude is 6."""
    m, e = math.frexp(amax)                  # amax = m * 2**e, m in [0.5, 1)
    s = e - 3                                # amax / 2**s = 8m in [4, 8)
    if 8 * m > 6:
        s += 1                               # (6, 8) -> (3, 4)
    return s


def _encode_terms(row: np.ndarray, n_terms: int = 8) -> np.ndarray:
    res = row.astype(np.float64).copy()
    out = np.zeros_like(res)
    for _ in range(n_terms):
        amax = float(np.abs(res).max())
        if amax == 0.0:
            break
        s = _scale_exp(amax)
        assert 3 < amax / 2.0 ** s <= 6
        codes = mxfp4.encode_e2m1(res, 127 + s)
        part = mxfp4.E2M1_TABLE[codes] * 2.0 ** s
        out += part
        res -= part
    return out


def test_scale_exponent_range():
    for amax in (1e-30, 0.37, 1.0, 3.0, 3.0000001, 5.99, 6.0, 6.01, 7.9, 1e30):
        s = _scale_exp(amax)
        assert 3 < amax / 2.0 ** s <= 6, amax


def test_eight_terms_reproduce_bf16_rows():
    key = synth.stream_key(4242, "x")
    n = 64 * 2048
    g = synth.normal_np(key, 0, n) * 3.0
    u = synth.normal_np(key, n, n) * 3.0
    h = mxfp4.round_bf16(g / (1.0 + np.exp(-g)) * u).reshape(64, 2048)
    x = mxfp4.round_bf16(synth.normal_np(key, 2 * n, 8 * 7168)).reshape(8, 7168)
    for rows in (h, x):
        rec = np.stack([_encode_terms(r) for r in rows])
        rel = np.linalg.norm(rec - rows) / np.linalg.norm(rows)
        exact = np.mean(rec == rows)
        assert rel < 1e-7, rel                 # the FFN tolerance is 2e-3
        assert exact > 0.99, exact


def test_fewer_terms_are_coarser():
    """Each term removes about two more bits: the error falls with the count."""
    key = synth.stream_key(4243, "x")
    row = mxfp4.round_bf16(synth.normal_np(key, 0, 2048))
    errs = [np.linalg.norm(_encode_terms(row, t) - row) for t in (2, 4, 6, 8)]
    assert errs[0] > errs[1] > errs[2] >= errs[3]

"""Pins of the oracle's greedy and rejection-sampling acceptance.

Greedy: brute force over every draft block of a tiny vocabulary, and the two
degenerate blocks.  Rejection: the special cases that the acceptance test
fixes exactly, the integer inverse-CDF draw at its boundaries, and the
losslessness the pages state, as a chi-square test of the emitted-token
marginal against the target distribution over 10**6 seeded trials -- with a
negative control that plants a mistake in the oracle and must fail.
"""
import itertools

import numpy as np
import pytest

from mxfp4_moe_block_b200 import synth
from oracle import accept


# ------------------------------------------------------------------ greedy --

def test_greedy_brute_force_all_drafts():
    rng = np.random.default_rng(0)
    S, K, V = 1, 3, 3
    for trial in range(20):
        logits = rng.integers(-2, 3, size=(S, K, V)).astype(np.float32)   # ties common
        am = [min(v for v in range(V) if logits[0, i, v] == logits[0, i].max()) for i in range(K)]
        for d in itertools.product(range(V), repeat=K):
            acc, nxt = accept.greedy(logits, np.array([d], np.int32))
            mism = [i for i in range(K) if d[i] != am[i]]
            a = mism[0] if mism else K
            assert acc[0] == a
            assert nxt[0] == (am[a] if a < K else -1)


def test_greedy_degenerate_blocks():
    rng = np.random.default_rng(1)
    S, K, V = 4, 8, 50
    logits = rng.standard_normal((S, K, V)).astype(np.float32)
    am = logits.argmax(axis=-1).astype(np.int32)
    acc, nxt = accept.greedy(logits, am)
    assert np.all(acc == K) and np.all(nxt == -1)
    bad = am.copy()
    bad[:, 0] = (bad[:, 0] + 1) % V
    acc, nxt = accept.greedy(logits, bad)
    assert np.all(acc == 0) and np.array_equal(nxt, am[:, 0])


# --------------------------------------------------------------- rejection --

def _one(p, q, x, ua, ur):
    p = np.asarray(p, np.float32)[None, None]
    q = np.asarray(q, np.float32)[None, None]
    return accept.rejection(p, q, np.array([[x]], np.int32),
                            np.array([[ua]], np.float32), np.array([ur], np.float32))


def test_rejection_equal_distributions_always_accept():
    p = np.array([0.25, 0.5, 0.25], np.float32)
    for x in range(3):
        for ua in (0.0, 0.5, 1.0 - 2.0 ** -24):
            acc, nxt = _one(p, p, x, ua, 0.3)
            assert acc[0] == 1 and nxt[0] == -1


def test_rejection_zero_q_and_zero_p():
    acc, _ = _one([0.5, 0.5], [1.0, 0.0], 1, 1.0 - 2.0 ** -24, 0.0)   # q(x)=0 < p(x): accept
    assert acc[0] == 1
    acc, nxt = _one([1.0, 0.0], [0.0, 1.0], 1, 0.0, 0.7)              # p(x)=0: reject
    assert acc[0] == 0 and nxt[0] == 0                                 # residual all on token 0


def test_rejection_threshold_is_exact():
    # accept iff u * q < p: with q = 0.5, p = 0.25 the boundary is u = 0.5
    acc, _ = _one([0.25, 0.75], [0.5, 0.5], 0, 0.5 - 2.0 ** -24, 0.0)
    assert acc[0] == 1
    acc, _ = _one([0.25, 0.75], [0.5, 0.5], 0, 0.5, 0.0)
    assert acc[0] == 0


def test_residual_integer_draw_boundaries():
    # residual r = (p - q)+ = [0.25, 0, 0.75] -> R = [2**38, 0, 3 * 2**38]
    p = np.array([0.5, 0.0, 0.75], np.float32)
    q = np.array([0.25, 0.5, 0.0], np.float32)
    # draws: m = floor(S*U/2**24) with S = 2**40; token 0 iff m < 2**38 iff U < 2**22
    assert accept.residual_sample(p, q, (2 ** 22 - 1) * 2.0 ** -24) == 0
    assert accept.residual_sample(p, q, 2 ** 22 * 2.0 ** -24) == 2
    assert accept.residual_sample(p, q, 0.0) == 0
    assert accept.residual_sample(p, q, 1.0 - 2.0 ** -24) == 2


def test_residual_falls_back_to_p_when_empty():
    p = np.array([0.5, 0.5], np.float32)
    assert accept.residual_sample(p, p, 0.75) == 1
    assert accept.residual_sample(p, p, 0.25) == 0


def test_rejection_first_reject_stops_the_block():
    V = 4
    p = np.zeros((1, 3, V), np.float32)
    q = np.zeros((1, 3, V), np.float32)
    p[0, :, 0] = 1.0
    q[0, :, 0] = 1.0
    p[0, 1] = [0.0, 1.0, 0.0, 0.0]          # row 1 rejects draft 0 (p=0)
    acc, nxt = accept.rejection(p, q, np.zeros((1, 3), np.int32),
                                np.zeros((1, 3), np.float32), np.array([0.5], np.float32))
    assert acc[0] == 1 and nxt[0] == 1


# ------------------------------------------------------ losslessness (chi2) --

CHI2_CRIT_15DOF_P001 = 37.697


def _chi2_trials(residual_fn=None, n=1_000_000, V=16, seed=77):
    """Emitted-token histogram of n single-token blocks, x ~ q."""
    zp = synth.normal_np(synth.stream_key(seed, "p_logits"), 0, V)
    zq = synth.normal_np(synth.stream_key(seed, "q_logits"), 0, V)
    p = np.exp(zp - zp.max()); p = (p / p.sum()).astype(np.float32)
    q = np.exp(zq - zq.max()); q = (q / q.sum()).astype(np.float32)
    ud = synth.u53_np(synth.stream_key(seed, "u_draft"), 0, n)
    x = synth.sample_rows_np(np.broadcast_to(q, (n, V)), ud)
    ua = synth.u24_np(synth.stream_key(seed, "u_accept"), 0, n).reshape(n, 1)
    ur = synth.u24_np(synth.stream_key(seed, "u_resample"), 0, n)
    P = np.broadcast_to(p, (n, 1, V))
    Q = np.broadcast_to(q, (n, 1, V))
    acc, nxt = accept.rejection(P, Q, x.reshape(n, 1), ua, ur)
    emitted = np.where(acc == 1, x, nxt)
    counts = np.bincount(emitted, minlength=V)
    expect = p.astype(np.float64) / p.astype(np.float64).sum() * n
    return float(((counts - expect) ** 2 / expect).sum())


def test_rejection_is_lossless_chi2():
    assert _chi2_trials() <= CHI2_CRIT_15DOF_P001


def test_rejection_negative_control_fails_chi2(monkeypatch):
    """Planting a mistake in the oracle (resample from p, not from the
    residual) must be caught by the same chi-square test."""
    real = accept.residual_sample

    def wrong(p_row, q_row, u):
        return real(p_row, np.zeros_like(q_row), u)
    monkeypatch.setattr(accept, "residual_sample", wrong)
    assert _chi2_trials() > CHI2_CRIT_15DOF_P001

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


# ------------------------------------------------------------ bonus row (K+1) --

def test_greedy_bonus_brute_force_all_drafts():
    """Every draft block over a 3-token vocabulary: the accepted prefix is the
    longest run of argmax matches and the emitted token is the argmax of the
    first unmatched row -- the bonus row K when all K match."""
    rng = np.random.default_rng(31)
    K, V = 3, 3
    logits = rng.normal(size=(1, K + 1, V)).astype(np.float32)
    am = logits[0].argmax(-1)
    for code in range(V ** K):
        d = np.array([(code // V ** i) % V for i in range(K)], np.int32)[None]
        acc, nxt = accept.greedy_bonus(logits, d)
        a = 0
        while a < K and d[0, a] == am[a]:
            a += 1
        assert acc[0] == a and nxt[0] == am[a]


def test_greedy_bonus_reduces_to_greedy_before_the_last_row():
    rng = np.random.default_rng(32)
    S, K, V = 64, 8, 50
    logits = rng.normal(size=(S, K + 1, V)).astype(np.float32)
    am = logits[:, :K].argmax(-1)
    d = np.where(rng.random((S, K)) < 0.1, (am + 1) % V, am).astype(np.int32)
    acc_b, nxt_b = accept.greedy_bonus(logits, d)
    acc, nxt = accept.greedy(logits[:, :K], d)
    assert np.array_equal(acc_b, acc)
    part = acc < K
    assert np.array_equal(nxt_b[part], nxt[part])
    assert np.array_equal(nxt_b[~part], logits[~part, K].argmax(-1))
    assert (~part).any() and part.any()


def test_rejection_bonus_reduces_to_rejection_and_draws_from_p():
    rng = np.random.default_rng(33)
    S, K, V = 200, 4, 12
    p = rng.random((S, K + 1, V)).astype(np.float32)
    p /= p.sum(-1, keepdims=True)
    q = p[:, :K].copy()                               # q == p: every draft accepted
    d = rng.integers(0, V, (S, K)).astype(np.int32)
    ua = rng.random((S, K)).astype(np.float32)
    ur = (rng.integers(0, 2 ** 24, S) / 2 ** 24).astype(np.float32)
    acc, nxt = accept.rejection_bonus(p, q, d, ua, ur)
    assert (acc == K).all()
    for s in range(S):
        assert nxt[s] == accept.bonus_sample(p[s, K], ur[s])
    q2 = rng.random((S, K, V)).astype(np.float32)
    q2 /= q2.sum(-1, keepdims=True)
    acc2, nxt2 = accept.rejection_bonus(p, q2, d, ua, ur)
    acc1, nxt1 = accept.rejection(p[:, :K], q2, d, ua, ur)
    assert np.array_equal(acc2, acc1)
    part = acc1 < K
    assert np.array_equal(nxt2[part], nxt1[part])


def test_bonus_sample_boundaries():
    p = np.zeros(5, np.float32)
    p[1], p[3] = 0.25, 0.75
    assert accept.bonus_sample(p, 0.0) == 1
    assert accept.bonus_sample(p, 0.25 - 2 ** -24) == 1
    assert accept.bonus_sample(p, 0.25) == 3
    assert accept.bonus_sample(p, 1 - 2 ** -24) == 3


def _bonus_chi2(draw_row, n=1_000_000, V=16, seed=78):
    """Chi-square of 10^6 bonus draws from `draw_row(p)` against p."""
    z = synth.normal_np(synth.stream_key(seed, "p_logits"), 0, V)
    p = np.exp(z - z.max())
    p = (p / p.sum()).astype(np.float32)
    ur = synth.u24_np(synth.stream_key(seed, "u_resample"), 0, n)
    row = draw_row(p)
    Pw = np.floor(row.astype(np.float64) * 2.0 ** 40).astype(np.int64)
    cum = np.cumsum(Pw)
    U = (ur.astype(np.float64) * 2 ** 24).astype(np.int64)
    m = (cum[-1].astype(object) * U.astype(object)) // 2 ** 24
    draws = np.searchsorted(cum, np.array(m, dtype=np.int64), side="right")
    # the vectorised draw is the oracle's rule: spot-check it against bonus_sample
    for i in range(0, n, n // 50):
        assert draws[i] == accept.bonus_sample(row, ur[i])
    counts = np.bincount(draws, minlength=V)
    expect = p.astype(np.float64) / p.astype(np.float64).sum() * n
    return float(((counts - expect) ** 2 / expect).sum())


def test_bonus_draw_follows_p_chi2():
    """The bonus token of fully accepted blocks is distributed as the target's
    row K: chi-square over 10^6 seeded draws, 15 dof, p >= 0.001."""
    assert _bonus_chi2(lambda p: p) <= CHI2_CRIT_15DOF_P001


def test_bonus_chi2_negative_control():
    """A planted mistake -- the draw taken from the neighbouring token's
    probability (an off-by-one row index) -- fails the same test."""
    assert _bonus_chi2(lambda p: np.roll(p, 1)) > CHI2_CRIT_15DOF_P001

"""Pins of the oracle's routing, permutation, expert FFN, combine and norm.

Routing and permutation are checked against brute force by Python's stable
sort on tiny inputs (a different algorithm from the oracle's rank count);
the FFN against closed forms that need no matrix product; combine and norm
against hand-derived values.
"""
import math

import numpy as np
import pytest

from oracle import moe, mxfp4


# ----------------------------------------------------------------- routing --

def _brute_topk(row, k):
    return sorted(range(len(row)), key=lambda i: (-float(row[i]), i))[:k]


@pytest.mark.parametrize("E", [1, 2, 3, 5, 8])
def test_route_matches_sorted_brute_force(E):
    rng = np.random.default_rng(E)
    for trial in range(200):
        # few distinct values -> many ties; include signed zeros
        pool = np.array([-1.5, -0.0, 0.0, 0.25, 2.0], dtype=np.float32)
        row = pool[rng.integers(0, len(pool), size=E)]
        for k in range(1, E + 1):
            idx, w, _ = moe.route_topk(row[None, :], k)
            assert list(idx[0]) == _brute_topk(row, k), (row, k)


def test_route_signed_zero_is_a_tie():
    row = np.array([[0.0, -0.0, -0.0, 0.0]], dtype=np.float32)
    idx, w, _ = moe.route_topk(row, 2)
    assert list(idx[0]) == [0, 1]
    assert list(w[0]) == [0.5, 0.5]


def test_route_weights_closed_form():
    rng = np.random.default_rng(11)
    l = rng.standard_normal((50, 6)).astype(np.float32)
    idx, w, _ = moe.route_topk(l, 1)
    assert np.all(w == 1.0)
    idx, w, w64 = moe.route_topk(l, 2)
    for t in range(50):
        a, b = float(l[t, idx[t, 0]]), float(l[t, idx[t, 1]])
        assert a >= b
        assert abs(w64[t, 0] - 1.0 / (1.0 + math.exp(b - a))) < 1e-15
        assert abs(w64[t, 1] - 1.0 / (1.0 + math.exp(a - b))) < 1e-15
    idx, w, w64 = moe.route_topk(l, 6)
    assert np.allclose(w64.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    assert np.all(np.diff(w64, axis=1) <= 0)        # descending logits -> descending weights


def test_route_rejects_bad_k():
    with pytest.raises(ValueError):
        moe.route_topk(np.zeros((1, 4), np.float32), 5)
    with pytest.raises(ValueError):
        moe.route_topk(np.zeros((1, 4), np.float32), 0)


# ------------------------------------------------------------- permutation --

def _check_perm(idx, E, off, sp, pr):
    flat = idx.reshape(-1)
    P = flat.size
    assert off[0] == 0 and off[E] == P and np.all(np.diff(off) >= 0)
    assert sorted(sp.tolist()) == list(range(P))
    assert np.array_equal(pr[sp], np.arange(P))
    for e in range(E):
        seg = sp[off[e]:off[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg) > 0)


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (3, 2, 4), (8, 2, 8), (5, 3, 16), (16, 8, 256)])
def test_permute_matches_stable_sort(T, k, E):
    rng = np.random.default_rng(T * 100 + E)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    off, sp, pr = moe.permute(idx, E)
    _check_perm(idx, E, off, sp, pr)
    want = sorted(range(T * k), key=lambda p: (int(idx.reshape(-1)[p]), p))
    assert sp.tolist() == want


def test_permute_empty_and_bad_index():
    off, sp, pr = moe.permute(np.zeros((0, 2), np.int32), 4)
    assert list(off) == [0] * 5 and sp.size == 0
    with pytest.raises(ValueError):
        moe.permute(np.array([[0, 4]], np.int32), 4)


# -------------------------------------------------------------- expert FFN --

def _const_weights(H, I, code, scale=127, code_down=None, scale_down=None):
    cd = code if code_down is None else code_down
    sd = scale if scale_down is None else scale_down
    w13c = mxfp4.pack_codes(np.full((2 * I, H), code, np.uint8))
    w13s = np.full((2 * I, H // 32), scale, np.uint8)
    w2c = mxfp4.pack_codes(np.full((H, I), cd, np.uint8))
    w2s = np.full((H, I // 32), sd, np.uint8)
    return w13c, w13s, w2c, w2s


def _bf16_rows(rng, n, H):
    return mxfp4.round_bf16(rng.standard_normal((n, H)))


def test_ffn_all_ones_closed_form():
    """Every weight 1.0: g = u = sum(x), h = bf16(silu(s)*s), y_m = I*h."""
    H, I = 64, 32
    rng = np.random.default_rng(1)
    x = _bf16_rows(rng, 3, H)
    h, y = moe.expert_ffn(x, *_const_weights(H, I, code=2), I)
    for r in range(3):
        s = math.fsum(x[r])
        hv = mxfp4.round_bf16(np.array([s / (1 + math.exp(-s)) * s]))[0]
        assert np.all(h[r] == hv)
        assert np.allclose(y[r], I * hv, rtol=1e-15, atol=0)


def test_ffn_negative_gate_and_scales():
    """Gate/up weights -1 at scale 2**1, down weights 0.5 at scale 2**-2."""
    H, I = 64, 64
    rng = np.random.default_rng(2)
    x = _bf16_rows(rng, 2, H)
    w = _const_weights(H, I, code=10, scale=128, code_down=1, scale_down=125)
    h, y = moe.expert_ffn(x, *w, I)
    for r in range(2):
        g = -2.0 * math.fsum(x[r])
        hv = mxfp4.round_bf16(np.array([g / (1 + math.exp(-g)) * g]))[0]
        assert np.all(h[r] == hv)
        assert np.allclose(y[r], I * hv * 0.125, rtol=1e-15, atol=0)


def test_ffn_zero_codes_give_zero():
    H, I = 64, 32
    x = _bf16_rows(np.random.default_rng(3), 4, H)
    h, y = moe.expert_ffn(x, *_const_weights(H, I, code=0), I)
    assert np.all(h == 0) and np.all(y == 0)


def test_ffn_single_weights_pick_single_products():
    """One nonzero gate, up and down weight select single products."""
    H, I = 64, 32
    rng = np.random.default_rng(4)
    x = _bf16_rows(rng, 1, H)
    w13 = np.zeros((2 * I, H), np.uint8)
    w2 = np.zeros((H, I), np.uint8)
    n0, c0, c1, m0 = 5, 17, 40, 9
    w13[n0, c0] = 7            # gate: 6.0
    w13[I + n0, c1] = 11       # up: -1.5
    w2[m0, n0] = 4             # down: 2.0
    w = (mxfp4.pack_codes(w13), np.full((2 * I, H // 32), 127, np.uint8),
         mxfp4.pack_codes(w2), np.full((H, I // 32), 126, np.uint8))   # down scale 0.5
    h, y = moe.expert_ffn(x, *w, I)
    g, u = 6.0 * x[0, c0], -1.5 * x[0, c1]
    hv = mxfp4.round_bf16(np.array([g / (1 + math.exp(-g)) * u]))[0]
    assert h[0, n0] == hv and np.count_nonzero(h) <= 1
    assert y[0, m0] == hv * 1.0 and np.count_nonzero(y) <= 1


def test_ffn_down_scale_linearity():
    """Raising every down-projection scale byte by one doubles y exactly."""
    H, I = 64, 64
    rng = np.random.default_rng(5)
    x = _bf16_rows(rng, 2, H)
    w13c = rng.integers(0, 256, (2 * I, H // 2), dtype=np.uint8)
    w13s = rng.integers(120, 131, (2 * I, H // 32)).astype(np.uint8)
    w2c = rng.integers(0, 256, (H, I // 2), dtype=np.uint8)
    w2s = rng.integers(120, 131, (H, I // 32)).astype(np.uint8)
    h1, y1 = moe.expert_ffn(x, w13c, w13s, w2c, w2s, I)
    h2, y2 = moe.expert_ffn(x, w13c, w13s, w2c, (w2s + 1).astype(np.uint8), I)
    assert np.array_equal(h1, h2) and np.array_equal(y2, 2 * y1)
    # out_cols selects columns of the same result
    _, y3 = moe.expert_ffn(x, w13c, w13s, w2c, w2s, I, out_cols=[3, 0, 63])
    assert np.allclose(y3, y1[:, [3, 0, 63]], rtol=1e-13, atol=0)


def test_moe_ffn_groups_pairs_by_expert():
    H, I, E, k, T = 64, 32, 4, 2, 5
    rng = np.random.default_rng(6)
    x = _bf16_rows(rng, T, H)
    W = {e: (rng.integers(0, 256, (2 * I, H // 2), dtype=np.uint8),
             rng.integers(124, 130, (2 * I, H // 32)).astype(np.uint8),
             rng.integers(0, 256, (H, I // 2), dtype=np.uint8),
             rng.integers(124, 130, (H, I // 32)).astype(np.uint8)) for e in range(E)}
    idx = np.array([[0, 3], [3, 1], [0, 1], [2, 0], [3, 2]], np.int32)
    off, sp, pr = moe.permute(idx, E)
    h, y = moe.moe_ffn(x, k, I, lambda e: W[e], off, sp)
    for p in range(T * k):
        t, e = p // k, int(idx.reshape(-1)[p])
        he, ye = moe.expert_ffn(x[t:t + 1], *W[e], I)
        # same expert, same token; only the BLAS summation order differs
        assert np.allclose(h[pr[p]], he[0], rtol=2.0 ** -7, atol=0)
        assert np.allclose(y[pr[p]], ye[0], rtol=1e-2, atol=1e-6 * np.abs(ye).max())


# ---------------------------------------------------------- combine, norm --

def test_combine_single_slot_is_rounding():
    y = np.random.default_rng(7).standard_normal((3, 16))
    out, acc = moe.combine(y, np.arange(3, dtype=np.int32), np.ones((3, 1), np.float32))
    assert np.array_equal(acc, y) and np.array_equal(out, mxfp4.round_bf16(y))


def test_combine_two_slots_and_residual():
    y = np.array([[1.0, 2.0], [4.0, -8.0]])
    w = np.array([[0.25, 0.75]], np.float32)
    res = np.array([[0.5, 0.5]])
    out, acc = moe.combine(y, np.array([1, 0], np.int32), w, res)
    # slot 0 -> row 1, slot 1 -> row 0
    assert acc.tolist() == [[0.25 * 4 + 0.75 * 1 + 0.5, 0.25 * -8 + 0.75 * 2 + 0.5]]


def test_rms_norm_constant_rows():
    x = np.array([[3.0] * 8, [-0.5] * 8])
    out = moe.rms_norm(x, eps=0.0)
    assert np.array_equal(out, np.array([[1.0] * 8, [-1.0] * 8]))

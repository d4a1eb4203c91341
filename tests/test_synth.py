"""The seeded generator: numpy and torch draws agree byte for byte, sub-ranges
are consistent, and the distributions have the stated support."""
import numpy as np
import torch

from mxfp4_moe_block_b200 import synth


def test_splitmix_reference_values():
    # SplitMix64 with state 0 (Steele, Lea and Flood 2014; Vigna's reference
    # splitmix64.c): the first outputs from seed 0 are these constants.
    h = synth.hash_np(0, 0, 3)
    assert [int(v) for v in h] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_numpy_and_torch_bytes_agree_cpu():
    key = synth.stream_key(5, "w13_codes", 2)
    a = synth.bytes_np(key, 8 * 1000, 4096)
    b = synth.bytes_torch(key, 8 * 1000, 4096, "cpu").numpy()
    assert np.array_equal(a, b)
    s1 = synth.int_range_np(key, 77, 5000, 120, 130)
    s2 = synth.int_range_torch(key, 77, 5000, 120, 130, "cpu").numpy()
    assert np.array_equal(s1, s2)


def test_subranges_are_consistent():
    key = synth.stream_key(9, "w2_codes")
    whole = synth.bytes_np(key, 0, 1000)
    assert np.array_equal(whole[24:500], synth.bytes_np(key, 24, 476))
    assert np.array_equal(whole[13:31], synth.bytes_np(key, 13, 18))


def test_distribution_support():
    key = synth.stream_key(1, "w13_scales")
    s = synth.int_range_np(key, 0, 200000, 120, 130)
    assert s.min() == 120 and s.max() == 130
    counts = np.bincount(s - 120)
    assert counts.min() > 0.9 * 200000 / 11
    u = synth.u24_np(key, 0, 100000)
    assert u.min() >= 0 and u.max() < 1 and np.all(u * 2 ** 24 == np.floor(u * 2 ** 24))
    z = synth.normal_np(key, 0, 200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    codes = synth.bytes_np(key, 0, 100000)
    nib = np.concatenate([codes & 15, codes >> 4])
    assert np.bincount(nib).min() > 0.9 * nib.size / 16


def test_weights_torch_match_numpy_slices():
    sh = synth.Shape("t", H=256, I=128, E=4, k=2, S=1, K=8, V=64, seed=3)
    w13c, w13s, w2c, w2s = synth.weights_torch(sh, 0, "cpu", chunk_experts=3)
    for e in range(sh.E):
        assert np.array_equal(w13c[e].numpy(), synth.weight_codes_np(sh, "w13", e))
        assert np.array_equal(w13s[e].numpy(), synth.weight_scales_np(sh, "w13", e))
        assert np.array_equal(w2c[e].numpy(), synth.weight_codes_np(sh, "w2", e))
        assert np.array_equal(w2s[e].numpy(), synth.weight_scales_np(sh, "w2", e))


def test_bf16_bits_match_torch():
    z = synth.normal_np(synth.stream_key(2, "x"), 0, 10000).astype(np.float32)
    mine = synth.f32_to_bf16_bits(z)
    ref = torch.from_numpy(z).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


def test_drafts_follow_rules():
    sh = synth.SHAPES["tiny"]
    lg = synth.block_logits(sh)
    d = synth.greedy_drafts(sh, lg)
    am = lg.argmax(-1)
    assert d.shape == (sh.S, sh.K) and d.dtype == np.int32
    assert 0 < (d != am).sum() < sh.K
    sh2 = synth.Shape("g", H=256, I=128, E=8, k=2, S=2000, K=8, V=1000, seed=4)
    lg2 = synth.normal_np(1, 0, sh2.S * sh2.K * sh2.V).astype(np.float32).reshape(sh2.S, sh2.K, sh2.V)
    d2 = synth.greedy_drafts(sh2, lg2)
    am2 = lg2.argmax(-1)
    match = (d2 == am2)
    prefix = np.where(match.all(1), sh2.K, np.argmin(match, 1))
    # Geometric(1/7) prefix truncated at K = 8: mean = 6 * (1 - (6/7)**8)
    assert abs(prefix.mean() - 6 * (1 - (6 / 7) ** 8)) < 0.15


def test_sequence_range_draws_equal_rows_of_the_full_draw():
    """Drawing only sequences s0..s1-1 (the oracle's bounded samples do) gives
    the same values as those rows of the full draw, for every recipe."""
    sh = synth.Shape("t", H=256, I=128, E=8, k=2, S=5, K=4, V=300, seed=9)
    full = synth.block_logits(sh)
    part = synth.block_logits(sh, seqs=(2, 4))
    assert np.array_equal(full[2:4], part)
    for rule in ("geometric", "perturb4"):
        assert np.array_equal(synth.greedy_drafts(sh, full, rule)[2:4],
                              synth.greedy_drafts(sh, part, rule, seqs=(2, 4)))
    for bonus in (False, True):
        r = synth.rejection_inputs(sh, bonus=bonus)
        rp = synth.rejection_inputs(sh, bonus=bonus, seqs=(1, 3))
        for a, b in zip((r.p, r.q, r.draft, r.u_accept, r.u_resample),
                        (rp.p, rp.q, rp.draft, rp.u_accept, rp.u_resample)):
            assert np.array_equal(a[1:3], b)
    lb = synth.block_logits(sh, rows=sh.K + 1)
    assert lb.shape == (sh.S, sh.K + 1, sh.V)
    assert np.array_equal(lb[3:5], synth.block_logits(sh, rows=sh.K + 1, seqs=(3, 5)))

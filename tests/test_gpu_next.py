"""GPU parity of the calls beyond the verify step's six: the bonus-row
acceptance variants and the MXFP4 weight quantiser, against the oracle on
the same seeded inputs.  All results are integers and must match bit for bit.
"""
import numpy as np
import pytest
import torch

import mxfp4_moe_block_b200 as mm
from mxfp4_moe_block_b200 import synth
from oracle import accept as oacc
from oracle import mxfp4 as omx

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def clean_status():
    mm.moe_clear_device_status()
    yield


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


# ------------------------------------------------------------ bonus rows --

@pytest.mark.parametrize("name", ["tiny", "batch1", "dflash16", "multilayer"])
def test_greedy_bonus_bit_exact(name):
    """Shapes of the seeded workloads with K+1 target rows; every other
    sequence drafts the target argmax throughout, so both the first-mismatch
    and the all-accepted (bonus token) outcomes occur."""
    sh = synth.SHAPES[name]
    if sh.S < 3:                 # room for both outcomes: 6 blocks of the same size
        sh = synth.Shape(**{**sh.__dict__, "S": 6})
    K = sh.K
    lg = synth.block_logits(sh, rows=K + 1)
    d = synth.greedy_drafts(sh, np.ascontiguousarray(lg[:, :K]))
    am = lg[:, :K].argmax(-1).astype(np.int32)
    d[::2] = am[::2]
    acc, nxt = mm.block_accept_greedy_bonus(_t(lg), _t(d))
    racc, rnxt = oacc.greedy_bonus(lg, d)
    assert np.array_equal(acc.cpu().numpy(), racc)
    assert np.array_equal(nxt.cpu().numpy(), rnxt)
    assert (racc == K).any() and (racc < K).any()
    assert mm.moe_get_device_status() == (0, 0)


def test_greedy_bonus_edges():
    """Ties, K = 1 and K = 32 (33 rows), ragged and tiny vocabularies."""
    rng = np.random.default_rng(21)
    for S, K, V in [(3, 1, 1), (4, 32, 1001), (7, 8, 7), (5, 3, 5000), (2, 16, 32000)]:
        lg = rng.integers(-3, 3, (S, K + 1, V)).astype(np.float32)
        am = lg[:, :K].argmax(-1).astype(np.int32)
        for d in (am, np.where(rng.random((S, K)) < 0.3, (am + 1) % V, am).astype(np.int32)):
            acc, nxt = mm.block_accept_greedy_bonus(_t(lg), _t(d))
            racc, rnxt = oacc.greedy_bonus(lg, d)
            assert np.array_equal(acc.cpu().numpy(), racc), (S, K, V)
            assert np.array_equal(nxt.cpu().numpy(), rnxt), (S, K, V)
    assert mm.moe_get_device_status() == (0, 0)


@pytest.mark.parametrize("name", ["tiny", "dflash16", "multilayer"])
def test_rejection_bonus_bit_exact(name):
    """Seeded rejection inputs with a bonus target row; every third sequence
    has q = p on its K rows, so all its drafts are accepted and the token is
    drawn from the bonus row."""
    sh = synth.SHAPES[name]
    if sh.S < 3:                 # room for both outcomes: 6 blocks of the same size
        sh = synth.Shape(**{**sh.__dict__, "S": 6})
    K = sh.K
    ri = synth.rejection_inputs(sh, bonus=True)
    q = ri.q.copy()
    q[::3] = ri.p[::3, :K]
    acc, nxt = mm.block_accept_rejection_bonus(_t(ri.p), _t(q), _t(ri.draft), _t(ri.u_accept),
                                               _t(ri.u_resample))
    racc, rnxt = oacc.rejection_bonus(ri.p, q, ri.draft, ri.u_accept, ri.u_resample)
    assert np.array_equal(acc.cpu().numpy(), racc)
    assert np.array_equal(nxt.cpu().numpy(), rnxt)
    assert (racc == K).any() and (racc < K).any()
    assert mm.moe_get_device_status() == (0, 0)


def test_rejection_bonus_row_without_mass_sets_status():
    p = torch.zeros((1, 2, 8), device=DEV)
    p[0, 0] = 0.125
    d = torch.tensor([[3]], dtype=torch.int32, device=DEV)
    ua = torch.zeros((1, 1), device=DEV)
    ur = torch.zeros(1, device=DEV)
    acc, nxt = mm.block_accept_rejection_bonus(p, p[:, :1].contiguous(), d, ua, ur)
    assert mm.moe_get_device_status() == (5, 2)
    assert acc.item() == 1 and nxt.item() == -1


def test_rejection_bonus_draw_chi2_on_gpu():
    """The bonus token follows the target's bonus row: 10**6 single-draft
    blocks with q = p on the verified row (so every draft is accepted), the
    bonus token counted against p[1] (chi-square, 15 dof, p >= 0.001)."""
    n, V, seed = 1_000_000, 16, 91
    z0 = synth.normal_np(synth.stream_key(seed, "p_logits"), 0, V)
    z1 = synth.normal_np(synth.stream_key(seed, "p_logits", 1), 0, V)
    p0 = np.exp(z0 - z0.max()); p0 = (p0 / p0.sum()).astype(np.float32)
    p1 = np.exp(z1 - z1.max()); p1 = (p1 / p1.sum()).astype(np.float32)
    x = synth.sample_rows_np(np.broadcast_to(p0, (n, V)),
                             synth.u53_np(synth.stream_key(seed, "u_draft"), 0, n))
    ua = synth.u24_np(synth.stream_key(seed, "u_accept"), 0, n).reshape(n, 1)
    ur = synth.u24_np(synth.stream_key(seed, "u_resample"), 0, n)
    P = torch.from_numpy(np.stack([p0, p1])).to(DEV).expand(n, 2, V).contiguous()
    Q = P[:, :1].contiguous()
    acc, nxt = mm.block_accept_rejection_bonus(P, Q, _t(x.reshape(n, 1)), _t(ua), _t(ur))
    acc, nxt = acc.cpu().numpy(), nxt.cpu().numpy()
    assert (acc == 1).all()
    counts = np.bincount(nxt, minlength=V)
    expect = p1.astype(np.float64) / p1.astype(np.float64).sum() * n
    chi2 = float(((counts - expect) ** 2 / expect).sum())
    assert chi2 <= 37.697, chi2


# -------------------------------------------------------------- quantiser --

def _bf16_bits(a):
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


def _adversarial_rows():
    """Blocks at the conversion's boundaries, as bf16 bit patterns [R, 128]:
    elements exactly at E2M1 midpoints (ties), amax a power of two and just
    below one, elements past 6 (saturation), zero and negative-zero blocks,
    bf16 subnormals, the largest bf16 and mixed signs."""
    rows = []
    for e in (-130, -126, -20, 0, 7, 100, 125):
        X = 2.0 ** e
        mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 4.0]) * X
        blk_ties = np.concatenate([mids, -mids, mids / 2, -mids * 1.0])[:32]
        blk_ties[7] = 4.0 * X                      # amax = 4X: the block's scale is X
        pow2 = np.full(32, 0.3 * X); pow2[5] = 4.0 * X
        below = np.full(32, 0.7 * X); below[9] = (2 - 2.0 ** -7) * 4.0 * X   # ratio ~7.97 -> 6
        sat = np.linspace(-7.9, 7.9, 32) * X
        sat[0] = 4.0 * X
        rows.append(np.concatenate([blk_ties, pow2, below, sat]))
    z = np.zeros(128); rows.append(z)
    rows.append(-z)                                # all negative zero
    sub = np.zeros(128); sub[::3] = 2.0 ** -133; sub[1::3] = -(2.0 ** -130); rows.append(sub)
    big = np.full(128, 1.0); big[::7] = 3.3895313892515355e38; big[1::7] = -1e38; rows.append(big)
    out = np.stack([_bf16_bits(r) for r in rows])
    neg0 = out[-4 + 1]                             # the -0 row keeps its sign bits
    assert (neg0 == 0x8000).all()
    return out


def _quantize_check(bits, what):
    w = torch.from_numpy(bits.astype(np.uint16).view(np.int16)).to(DEV).view(torch.bfloat16)
    codes, scales = mm.mxfp4_quantize(w)
    rc, rs = omx.quantize_mxfp4(synth.bf16_bits_to_f32(bits).astype(np.float64))
    assert np.array_equal(scales.cpu().numpy(), rs), f"{what}: scales differ"
    assert np.array_equal(codes.cpu().numpy(), rc), f"{what}: codes differ"


def test_quantize_adversarial_blocks_bit_exact():
    _quantize_check(_adversarial_rows(), "adversarial")


@pytest.mark.parametrize("R,K,sd", [(64, 4096, 1.0), (33, 7168, 1e-3), (5, 32, 1e5), (128, 2048, 3e-39)])
def test_quantize_random_bit_exact(R, K, sd):
    """Normal weights with a random per-row magnitude, several tiles and a
    ragged last CTA."""
    key = synth.stream_key(R * 7 + K, "w13_codes")
    z = synth.normal_np(key, 0, R * K).reshape(R, K)
    row = np.exp2(synth.int_range_np(key, 0, R, 0, 16) - 8.0).reshape(R, 1)
    _quantize_check(_bf16_bits(z * row * sd), f"R={R} K={K}")


def test_quantize_full_expert_sampled_rows():
    """One expert's W13 at the verify workload's size ([2I, H] = [4096, 7168]):
    sampled rows against the oracle, and every block's round trip within the
    format's error bound (half the gap at the code, or saturation past 6)."""
    R, K = 4096, 7168
    key = synth.stream_key(4242, "w13_codes")
    z = synth.normal_np(key, 0, R * K).reshape(R, K) * 0.02
    bits = _bf16_bits(z)
    w = torch.from_numpy(bits.view(np.int16)).to(DEV).view(torch.bfloat16)
    codes, scales = mm.mxfp4_quantize(w)
    cg, sg = codes.cpu().numpy(), scales.cpu().numpy()
    rows = synth.int_range_np(key, 7, 48, 0, R - 1)
    for r in rows:
        rc, rs = omx.quantize_mxfp4(synth.bf16_bits_to_f32(bits[r:r + 1]).astype(np.float64))
        assert np.array_equal(sg[r:r + 1], rs) and np.array_equal(cg[r:r + 1], rc), r
    # every row: the dequantised values stay within one E2M1 step of the input
    deq = omx.dequantize(cg[:256], sg[:256])
    x = synth.bf16_bits_to_f32(bits[:256]).astype(np.float64)
    step = np.repeat(np.ldexp(1.0, sg[:256].astype(np.int64) - 127), 32, axis=1)
    assert np.all(np.abs(deq - x) <= 2.0 * step)


def test_quantize_argument_errors():
    L = mm.lib()
    assert L.mxfp4_quantize(None, 4, 48, None, None, None) == 1          # K % 32
    assert L.mxfp4_quantize(None, -1, 64, None, None, None) == 1
    assert L.mxfp4_quantize(None, 0, 64, None, None, None) == 0          # empty
    w = torch.zeros((2, 64), dtype=torch.bfloat16, device=DEV)
    c = torch.empty(2 * 32 + 4, dtype=torch.uint8, device=DEV)
    s = torch.empty(4, dtype=torch.uint8, device=DEV)
    # misaligned codes pointer
    assert L.mxfp4_quantize(w.data_ptr(), 2, 64, c.data_ptr() + 1, s.data_ptr(),
                            torch.cuda.current_stream().cuda_stream) == 1

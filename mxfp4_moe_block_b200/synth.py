"""Seeded synthetic inputs for the MXFP4 MoE block-verify path.

This module draws random numbers only. It holds none of the method's
arithmetic (no decoding, routing, FFN or acceptance), so that both the CUDA
path and the CPU oracle can be fed the very same bytes without sharing any
computation.

Generator: a counter-based hash. Element ``i`` of a stream with 64-bit key
``K`` is ``mix64(K + (i + 1) * GOLDEN mod 2**64)``, where ``mix64`` is the
SplitMix64 output finaliser (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014; constants of Stafford's
"Mix13").  Because element ``i`` depends on ``i`` alone, any sub-range of a
tensor can be drawn on its own (the oracle draws only the experts it needs)
and the device implementation (torch integer ops) gives identical bytes.

Distributions (all fixed here, nowhere else):
  * bytes          : the 8 little-endian bytes of one hash per 8 output bytes
  * scale in [lo,hi]: lo + (((h >> 32) * (hi - lo + 1)) >> 32)
  * uniform u24    : (h >> 40) * 2**-24, an exact float32 in [0, 1)
  * uniform u53    : (h >> 11) * 2**-53 (float64, for inverse-CDF draws)
  * normal N(0,1)  : Box-Muller on two independent streams, float64
  * bf16 values    : float64 -> float32 (round to nearest even) -> bf16 (RNE)

Workload recipes for the five shapes of the block-verify problem live in
:func:`make_block`, :func:`make_layer` and friends below.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_SPLIT_B = 0xD1B54A32D192ED03

# Stream tags: one per tensor kind.
TAG = {
    "x": 1, "router": 2, "router_bias": 3,
    "w13_codes": 4, "w13_scales": 5, "w2_codes": 6, "w2_scales": 7,
    "block_logits": 8, "draft_perturb": 9, "draft_pos": 10, "geom": 11,
    "p_logits": 12, "q_logits": 13, "u_draft": 14, "u_accept": 15,
    "u_resample": 16, "draft_random": 17,
}


def _mix64_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * _M1) & MASK64
    z = ((z ^ (z >> 27)) * _M2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tag: str, layer: int = 0, sub: int = 0) -> int:
    """64-bit key of the stream (seed, tensor kind, layer, sub-stream)."""
    k = _mix64_int(seed * GOLDEN + 0x5EED)
    k = _mix64_int(k ^ (TAG[tag] * GOLDEN & MASK64))
    k = _mix64_int(k ^ ((layer + 1) * _M1 & MASK64))
    if sub:
        k = _mix64_int(k ^ (sub * _SPLIT_B & MASK64))
    return k


# --------------------------------------------------------------------------
# numpy (CPU) implementation
# --------------------------------------------------------------------------

def hash_np(key: int, start: int, count: int) -> np.ndarray:
    """uint64 hashes of elements [start, start+count) of stream ``key``."""
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        z = np.uint64(key) + i * np.uint64(GOLDEN)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_M1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_M2)
        return z ^ (z >> np.uint64(31))


def bytes_np(key: int, start_byte: int, nbytes: int) -> np.ndarray:
    """Bytes [start_byte, start_byte+nbytes) of a byte stream (8 per hash)."""
    h0 = start_byte // 8
    h1 = (start_byte + nbytes + 7) // 8
    b = hash_np(key, h0, h1 - h0).astype("<u8").view(np.uint8)
    off = start_byte - h0 * 8
    return b[off:off + nbytes].copy()


def int_range_np(key: int, start: int, count: int, lo: int, hi: int) -> np.ndarray:
    """Integers uniform in [lo, hi] (multiply-shift of the top 32 bits)."""
    h = hash_np(key, start, count)
    span = np.uint64(hi - lo + 1)
    return (np.uint64(lo) + (((h >> np.uint64(32)) * span) >> np.uint64(32))).astype(np.int64)


def u24_np(key: int, start: int, count: int) -> np.ndarray:
    """Uniform float32 in [0,1), multiples of 2**-24."""
    h = hash_np(key, start, count)
    return ((h >> np.uint64(40)).astype(np.float64) * 2.0 ** -24).astype(np.float32)


def u53_np(key: int, start: int, count: int) -> np.ndarray:
    h = hash_np(key, start, count)
    return (h >> np.uint64(11)).astype(np.float64) * 2.0 ** -53


def normal_np(key: int, start: int, count: int) -> np.ndarray:
    """Standard normal float64 by Box-Muller over two sub-streams."""
    ha = hash_np(key, start, count)
    hb = hash_np(_mix64_int(key ^ _SPLIT_B), start, count)
    u1 = ((ha >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53  # (0, 1]
    u2 = (hb >> np.uint64(11)).astype(np.float64) * 2.0 ** -53          # [0, 1)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rnd = ((u >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
    return ((u + rnd) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# torch implementation of the byte/scale streams (runs on any device)
# --------------------------------------------------------------------------

def _s64(v: int) -> int:
    v &= MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _lsr(t, s: int):
    return (t >> s) & ((1 << (64 - s)) - 1)


def hash_torch(key: int, start: int, count: int, device):
    import torch
    i = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    z = i * _s64(GOLDEN) + _s64(key)
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def bytes_torch(key: int, start_byte: int, nbytes: int, device, out=None):
    """Same bytes as :func:`bytes_np`; ``start_byte`` must be a multiple of 8."""
    import torch
    assert start_byte % 8 == 0
    nh = (nbytes + 7) // 8
    b = hash_torch(key, start_byte // 8, nh, device).view(torch.uint8)[:nbytes]
    if out is None:
        return b.clone()
    out.copy_(b)
    return out


def int_range_torch(key: int, start: int, count: int, lo: int, hi: int, device):
    h = hash_torch(key, start, count, device)
    return lo + ((_lsr(h, 32) * (hi - lo + 1)) >> 32)


# --------------------------------------------------------------------------
# Workload shapes
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class Shape:
    """One MoE verify workload: S sequences x K-token blocks, top-k of E."""
    name: str
    H: int
    I: int
    E: int
    k: int
    S: int
    K: int
    V: int
    layers: int = 1
    accept: tuple = ("greedy",)
    router_bias_sd: float = 0.0
    draft_rule: str = "geometric"   # 'perturb4' | 'geometric' | 'from_q'
    scale_lo: int = 120
    scale_hi: int = 130
    seed: int = 1000

    @property
    def T(self) -> int:
        return self.S * self.K

    @property
    def P(self) -> int:
        return self.T * self.k

    def expert_bytes(self) -> int:
        """Codes + scales of one expert's three matrices."""
        H, I = self.H, self.I
        return 2 * I * (H // 2 + H // 32) + H * (I // 2 + I // 32)


SHAPES = {
    "tiny": Shape("tiny", H=256, I=128, E=8, k=2, S=1, K=8, V=1024,
                  draft_rule="perturb4", seed=1000),
    "batch1": Shape("batch1", H=7168, I=2048, E=256, k=8, S=1, K=8, V=152064,
                    draft_rule="geometric", seed=1001),
    "serving": Shape("serving", H=7168, I=2048, E=256, k=8, S=16, K=8, V=152064,
                     router_bias_sd=0.5, draft_rule="geometric", seed=1002),
    "dflash16": Shape("dflash16", H=4096, I=1536, E=128, k=8, S=64, K=16, V=32000,
                      accept=("rejection",), draft_rule="from_q", seed=1003),
    "multilayer": Shape("multilayer", H=7168, I=2048, E=256, k=8, S=32, K=8, V=152064,
                        layers=8, accept=("greedy", "rejection"),
                        draft_rule="geometric", seed=1004),
}


# ---- per-tensor recipes (numpy; small tensors are always drawn on the CPU) --

def x_bf16_bits(sh: Shape, layer: int = 0) -> np.ndarray:
    """Activations x [T, H]: bf16(N(0,1)) as uint16 bit patterns."""
    z = normal_np(stream_key(sh.seed, "x", layer), 0, sh.T * sh.H)
    return f32_to_bf16_bits(z.astype(np.float32)).reshape(sh.T, sh.H)


def router_logits(sh: Shape, layer: int = 0) -> np.ndarray:
    """Router logits [T, E] float32: N(0,1), plus a per-expert N(0, sd) bias."""
    z = normal_np(stream_key(sh.seed, "router", layer), 0, sh.T * sh.E).reshape(sh.T, sh.E)
    if sh.router_bias_sd > 0:
        b = sh.router_bias_sd * normal_np(stream_key(sh.seed, "router_bias", layer), 0, sh.E)
        z = z + b[None, :]
    return z.astype(np.float32)


def weight_codes_np(sh: Shape, which: str, expert: int, layer: int = 0) -> np.ndarray:
    """Packed E2M1 codes of one expert: w13 [2I, H/2] or w2 [H, I/2] uint8."""
    rows, cols = (2 * sh.I, sh.H // 2) if which == "w13" else (sh.H, sh.I // 2)
    per = rows * cols
    b = bytes_np(stream_key(sh.seed, which + "_codes", layer), expert * per, per)
    return b.reshape(rows, cols)


def weight_scales_np(sh: Shape, which: str, expert: int, layer: int = 0) -> np.ndarray:
    """E8M0 scale bytes of one expert: w13 [2I, H/32] or w2 [H, I/32] uint8."""
    rows, cols = (2 * sh.I, sh.H // 32) if which == "w13" else (sh.H, sh.I // 32)
    per = rows * cols
    s = int_range_np(stream_key(sh.seed, which + "_scales", layer), expert * per, per,
                     sh.scale_lo, sh.scale_hi)
    return s.astype(np.uint8).reshape(rows, cols)


def weights_torch(sh: Shape, layer: int, device, chunk_experts: int = 8):
    """All experts' codes and scales of one layer, drawn on ``device``.

    Returns (w13_codes [E,2I,H/2], w13_scales [E,2I,H/32], w2_codes [E,H,I/2],
    w2_scales [E,H,I/32]) as uint8 tensors, byte-identical to the numpy draws.
    """
    import torch
    out = []
    for which in ("w13", "w2"):
        rows, cols = (2 * sh.I, sh.H) if which == "w13" else (sh.H, sh.I)
        codes = torch.empty((sh.E, rows, cols // 2), dtype=torch.uint8, device=device)
        scales = torch.empty((sh.E, rows, cols // 32), dtype=torch.uint8, device=device)
        kc = stream_key(sh.seed, which + "_codes", layer)
        ks = stream_key(sh.seed, which + "_scales", layer)
        per_c = rows * cols // 2
        per_s = rows * cols // 32
        flat_c = codes.view(-1)
        flat_s = scales.view(-1)
        for e0 in range(0, sh.E, chunk_experts):
            e1 = min(sh.E, e0 + chunk_experts)
            bytes_torch(kc, e0 * per_c, (e1 - e0) * per_c, device,
                        out=flat_c[e0 * per_c:e1 * per_c])
            flat_s[e0 * per_s:e1 * per_s].copy_(
                int_range_torch(ks, e0 * per_s, (e1 - e0) * per_s,
                                sh.scale_lo, sh.scale_hi, device).to(torch.uint8))
        out += [codes, scales]
    return tuple(out)


def _target_argmax(logits: np.ndarray) -> np.ndarray:
    # Workload construction only: which token the drafts should copy.
    return np.argmax(logits, axis=-1)


def _seq_range(sh: Shape, seqs) -> tuple:
    s0, s1 = (0, sh.S) if seqs is None else seqs
    if not 0 <= s0 < s1 <= sh.S:
        raise ValueError("sequence range outside [0, S)")
    return s0, s1


def block_logits(sh: Shape, layer: int = 0, rows: int | None = None, seqs=None) -> np.ndarray:
    """Target logits [S, R, V] float32: N(0, 2) (2 = standard deviation).

    R = K by default; R = K + 1 draws blocks with a bonus row (the target's
    scores for the position after the block).  ``seqs`` = (s0, s1) draws
    only those sequences (the same values as rows s0..s1-1 of the full draw)."""
    R = sh.K if rows is None else rows
    s0, s1 = _seq_range(sh, seqs)
    z = normal_np(stream_key(sh.seed, "block_logits", layer), s0 * R * sh.V, (s1 - s0) * R * sh.V)
    return (2.0 * z).astype(np.float32).reshape(s1 - s0, R, sh.V)


def greedy_drafts(sh: Shape, logits: np.ndarray, rule: str | None = None,
                  seqs=None) -> np.ndarray:
    """Draft tokens [S, K] int32 built around the target argmax.

    'perturb4'  : each position independently replaced w.p. 1/4 by
                  (argmax + 1 + r) mod V, r uniform in [0, V-2].
    'geometric' : a prefix of length L ~ Geometric(1/7) on {0,1,...} (mean 6)
                  copies the argmax, position L (if < K) is perturbed as
                  above, later positions are uniform over the vocabulary.
    """
    rule = rule or sh.draft_rule
    K, V = sh.K, sh.V
    s0, s1 = _seq_range(sh, seqs)
    S = s1 - s0
    am = _target_argmax(logits).astype(np.int64)
    r = int_range_np(stream_key(sh.seed, "draft_perturb"), s0 * K, S * K, 0, V - 2).reshape(S, K)
    pert = (am + 1 + r) % V
    if rule == "perturb4":
        pick = int_range_np(stream_key(sh.seed, "draft_pos"), s0 * K, S * K, 0, 3).reshape(S, K) == 0
        d = np.where(pick, pert, am)
    else:
        u = u53_np(stream_key(sh.seed, "geom"), s0, S)
        # inverse CDF of Geometric(p) on {0,1,...}: floor(log(1-u)/log(1-p))
        L = np.floor(np.log1p(-u) / math.log1p(-1.0 / 7.0)).astype(np.int64)
        rnd = int_range_np(stream_key(sh.seed, "draft_random"), s0 * K, S * K, 0, V - 1).reshape(S, K)
        pos = np.arange(K)[None, :]
        d = np.where(pos < L[:, None], am, np.where(pos == L[:, None], pert, rnd))
    return d.astype(np.int32)


def _softmax64(z: np.ndarray) -> np.ndarray:
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=-1, keepdims=True)


@dataclass
class RejectionInputs:
    p: np.ndarray          # [S, K, V] float32 target probabilities
    q: np.ndarray          # [S, K, V] float32 draft probabilities
    draft: np.ndarray      # [S, K] int32, drawn from q
    u_accept: np.ndarray   # [S, K] float32 (multiples of 2**-24)
    u_resample: np.ndarray # [S] float32 (multiples of 2**-24)


def rejection_inputs(sh: Shape, layer: int = 0, bonus: bool = False,
                     seqs=None) -> RejectionInputs:
    """p, q = softmax of independent N(0,2) logits; drafts x_i ~ q_i.

    With ``bonus`` p has K + 1 rows per sequence (row K: the target after the
    block); q and the drafts keep K.  ``seqs`` = (s0, s1) draws only those
    sequences (the same values as rows s0..s1-1 of the full draw)."""
    K, V = sh.K, sh.V
    s0, s1 = _seq_range(sh, seqs)
    S = s1 - s0
    n = S * K * V
    Kp = K + 1 if bonus else K
    zp = 2.0 * normal_np(stream_key(sh.seed, "p_logits", layer), s0 * Kp * V,
                         S * Kp * V).reshape(S, Kp, V)
    zq = 2.0 * normal_np(stream_key(sh.seed, "q_logits", layer), s0 * K * V, n).reshape(S, K, V)
    p = _softmax64(zp).astype(np.float32)
    q = _softmax64(zq).astype(np.float32)
    draft = sample_rows_np(q, u53_np(stream_key(sh.seed, "u_draft", layer), s0 * K,
                                     S * K).reshape(S, K))
    ua = u24_np(stream_key(sh.seed, "u_accept", layer), s0 * K, S * K).reshape(S, K)
    ur = u24_np(stream_key(sh.seed, "u_resample", layer), s0, S)
    return RejectionInputs(p, q, draft, ua, ur)


def sample_rows_np(prob: np.ndarray, u: np.ndarray) -> np.ndarray:
    """Inverse-CDF draw of one index per row of ``prob`` (float64 cumsum)."""
    c = np.cumsum(prob.astype(np.float64), axis=-1)
    t = u * c[..., -1]
    idx = (c <= t[..., None]).sum(axis=-1)
    return np.minimum(idx, prob.shape[-1] - 1).astype(np.int32)

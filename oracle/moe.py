"""MoE verify layer: route, permute, expert FFN, combine (oracle; test infra).

What the pages fix: the target model verifies a drafted block in one forward
pass ([P2] "如何评价小米6月9日发布的MiMo-V2.5-Pro-UltraSpeed模式？", section
"二、投机解码"; [P3] "MiMo-v2.5-Pro-UltraSpeed - infra 架构解读", section
"数据流概览") through MoE layers whose experts hold MXFP4 weights while the
router keeps higher precision ([P1] "mimo-v2-5-speculative-decoding-draft-
scheduling", section "接受率预测与动态回退机制"; [P4] "mimo-tilert-1000tps-
trillion-parameter-inference", sections "万亿参数推理为什么特别难" and
"第一层：FP4 选择性量化").  Each token activates a few experts ([P4],
"万亿参数推理为什么特别难").  The pages leave the routing function, the expert
FFN and the combine unstated; the readings used here are:

* top-k of the given fp32 router logits, ties to the lowest expert index,
  weights = softmax over the k selected logits (computed in float64, rounded
  once to float32);
* pairs p = t*k + j grouped by expert, ascending p inside an expert (stable);
* SwiGLU expert FFN, gate rows 0..I-1 and up rows I..2I-1 of one [2I, H]
  MXFP4 matrix, down matrix [H, I]; activations bf16, the SwiGLU output h
  rounded to bf16 before the down projection, y kept at full precision;
* out[t] = bf16(sum_j w[t,j] * y[t,j] (+ residual[t])) in slot order;
* between stacked layers a parameter-free RMSNorm (eps 1e-6) of the bf16
  residual stream feeds the next layer's experts.
"""
from __future__ import annotations

import numpy as np

from .mxfp4 import dequantize, round_bf16


# ----------------------------------------------------------------- routing --

def route_topk(logits: np.ndarray, k: int):
    """Top-k experts per token and their weights.

    Selection by rank: expert i of token t has rank
        r_i = #{ j : l_j > l_i  or  (l_j == l_i and j < i) }
    and is selected iff r_i < k; the selected experts are listed in rank
    order.  (Signed zeros compare equal and so tie.)  Weights are
        w_i = exp(l_i - l_max) / sum_{selected} exp(l_j - l_max)
    in float64, rounded once to float32.

    Returns topk_idx [T, k] int32, topk_w [T, k] float32 and the float64
    weights before rounding (for the rounding-boundary check in tests).
    """
    l = np.asarray(logits, dtype=np.float32)
    T, E = l.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    if not np.all(np.isfinite(l)):
        raise ValueError("router logits must be finite")
    idx = np.empty((T, k), dtype=np.int32)
    w64 = np.empty((T, k), dtype=np.float64)
    j = np.arange(E)
    for t in range(T):
        v = l[t].astype(np.float64)
        greater = v[None, :] > v[:, None]                      # [i, j]: l_j > l_i
        tie_lower = (v[None, :] == v[:, None]) & (j[None, :] < j[:, None])
        rank = (greater | tie_lower).sum(axis=1)
        for i in range(E):
            if rank[i] < k:
                idx[t, rank[i]] = i
        sel = v[idx[t]]
        ex = np.exp(sel - sel.max())
        w64[t] = ex / ex.sum()
    return idx, w64.astype(np.float32), w64


# ------------------------------------------------------------- permutation --

def permute(topk_idx: np.ndarray, E: int):
    """Group the pairs p = t*k + j by expert, stably.

    Returns expert_offsets [E+1] (exclusive prefix of per-expert counts),
    sorted_pair [P] (pair ids, expert-major, ascending inside an expert) and
    pair_row [P] (pair id -> its position in sorted_pair).
    """
    flat = np.asarray(topk_idx, dtype=np.int64).reshape(-1)
    P = flat.size
    if P and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert index out of range")
    offsets = np.zeros(E + 1, dtype=np.int32)
    sorted_pair = np.empty(P, dtype=np.int32)
    pos = 0
    for e in range(E):
        offsets[e] = pos
        for p in range(P):
            if flat[p] == e:
                sorted_pair[pos] = p
                pos += 1
    offsets[E] = pos
    pair_row = np.empty(P, dtype=np.int32)
    pair_row[sorted_pair] = np.arange(P, dtype=np.int32)
    return offsets, sorted_pair, pair_row


# -------------------------------------------------------------- expert FFN --

def silu(z: np.ndarray) -> np.ndarray:
    """z * sigmoid(z) = z / (1 + exp(-z)), float64."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def expert_ffn(xe: np.ndarray, w13_codes, w13_scales, w2_codes, w2_scales,
               I: int, out_cols=None):
    """SwiGLU FFN of one expert for a stack of token rows.

    xe: [n, H] float64 (bf16 values).  Returns h [n, I] (bf16 values as
    float64) and y [n, H] float64 (or only the columns in ``out_cols``):
        g = xe @ Wg^T,  u = xe @ Wu^T,  h = bf16(silu(g) * u),  y = h @ Wd^T
    with Wg, Wu the first and last I rows of the dequantised [2I, H] matrix.
    """
    w13 = dequantize(w13_codes, w13_scales)                    # [2I, H]
    g = xe @ w13[:I].T
    u = xe @ w13[I:].T
    h = round_bf16(silu(g) * u)
    if out_cols is None:
        wd = dequantize(w2_codes, w2_scales)                   # [H, I]
    else:
        cols = np.asarray(out_cols)
        wd = dequantize(w2_codes[cols], w2_scales[cols])
    y = h @ wd.T
    return h, y


def moe_ffn(x: np.ndarray, k: int, I: int, expert_weights, offsets, sorted_pair):
    """Expert FFN for every permuted pair.

    x: [T, H] float64; expert_weights(e) -> (w13_codes, w13_scales, w2_codes,
    w2_scales) of expert e.  Returns h [P, I] and y [P, H], both in
    sorted-row order (row r belongs to pair sorted_pair[r]).
    """
    E = len(offsets) - 1
    P = int(offsets[-1])
    H = x.shape[1]
    h = np.zeros((P, I))
    y = np.zeros((P, H))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r0 == r1:
            continue
        toks = np.asarray(sorted_pair[r0:r1]) // k
        he, ye = expert_ffn(x[toks], *expert_weights(e), I)
        h[r0:r1] = he
        y[r0:r1] = ye
    return h, y


# ---------------------------------------------------------------- combine --

def combine(y: np.ndarray, pair_row: np.ndarray, topk_w: np.ndarray,
            residual: np.ndarray | None = None):
    """out[t] = bf16( sum_j w[t,j] * y[pair_row[t*k+j]] + residual[t] ).

    Sum in float64 over slots j = 0..k-1.  Returns (bf16 values as float64,
    float64 values before rounding).
    """
    T, k = topk_w.shape
    acc = np.zeros((T, y.shape[1]))
    for t in range(T):
        for j in range(k):
            acc[t] += float(topk_w[t, j]) * y[pair_row[t * k + j]]
    if residual is not None:
        acc += residual
    return round_bf16(acc), acc


def rms_norm(x: np.ndarray, eps: float = 1e-6):
    """Parameter-free RMSNorm of bf16 rows: bf16(x / sqrt(mean(x^2) + eps))."""
    x = np.asarray(x, dtype=np.float64)
    r = np.sqrt((x * x).mean(axis=1, keepdims=True) + eps)
    return round_bf16(x / r)

"""Block acceptance: greedy prefix and rejection sampling (oracle; test infra).

Greedy ([P2] "如何评价小米6月9日发布的MiMo-V2.5-Pro-UltraSpeed模式？",
section "二、投机解码"): the tokens the target confirms are output, and from the
first wrong draft token on the target takes over.  Read here as: row i of the
target's logits checks draft token i; the accepted length a is the largest
prefix whose drafts equal the target argmax (ties to the lowest token id);
if a < K the target's own argmax at row a is emitted as the correction.

Rejection sampling ([P3] "MiMo-v2.5-Pro-UltraSpeed - infra 架构解读", section
"数据流概览", which names rejection sampling for the verify step; [P2], section
"六、效果如何", which states that accepted output is exactly what the target
would have produced): draft token x_i is accepted with probability
min(1, p_i(x_i)/q_i(x_i)); on the first rejection a token is drawn from the
residual distribution norm(max(0, p - q)).  The pages print no rule beyond
this; the exact-arithmetic reading used here (identical on every device):

* accept iff  double(u_i) * double(q_i[x_i]) < double(p_i[x_i])
  (the product of two float32 values is exact in float64);
* r_v = max(0, p_v - q_v) as one float32 subtraction, R_v = floor(r_v * 2**40)
  as an unsigned integer, S = sum_v R_v;
* with U = u_resample * 2**24 (an integer) the target mass is
  m = floor(S * U / 2**24) and the emitted token is the least v with
  R_0 + ... + R_v > m;
* if S == 0 the same draw is taken from P_v = floor(p_v * 2**40);
* all K accepted -> next token -1 (no bonus row).

With a bonus row (the K+1 convention of speculative decoding: the target also
scores the position after the block), all K accepted emits the target's own
token for that position instead of -1: its argmax (greedy), or a draw from p
at row K by the same integer rule on P_v (rejection).  `greedy_bonus` and
`rejection_bonus` state that variant.
"""
from __future__ import annotations

import numpy as np


def argmax_lowest(row: np.ndarray) -> int:
    """Index of the largest value; the lowest such index on ties."""
    return int(np.argmax(row))       # numpy returns the first occurrence


def greedy(logits: np.ndarray, draft: np.ndarray):
    """Greedy prefix acceptance.  logits [S, K, V], draft [S, K].

    Returns accept_len [S] int32 in [0, K] and next_token [S] int32
    (argmax of row accept_len, or -1 when every draft was accepted).
    """
    S, K, _ = logits.shape
    acc = np.zeros(S, dtype=np.int32)
    nxt = np.zeros(S, dtype=np.int32)
    for s in range(S):
        a = K
        for i in range(K):
            if argmax_lowest(logits[s, i]) != int(draft[s, i]):
                a = i
                break
        acc[s] = a
        nxt[s] = argmax_lowest(logits[s, a]) if a < K else -1
    return acc, nxt


def _draw(weights: list, U: int) -> int:
    """Least v with weights[0] + ... + weights[v] > floor(sum * U / 2**24)."""
    total = sum(weights)
    m = (total * U) >> 24
    run = 0
    for v, wv in enumerate(weights):
        run += wv
        if run > m:
            return v
    raise AssertionError("unreachable: m < total")


def residual_sample(p_row: np.ndarray, q_row: np.ndarray, u_resample: float) -> int:
    """Token drawn from norm(max(0, p - q)) with the exact integer rule."""
    r = np.maximum(p_row.astype(np.float32) - q_row.astype(np.float32), np.float32(0))
    R = [int(v) for v in np.floor(r.astype(np.float64) * 2.0 ** 40)]
    U = int(float(u_resample) * 2 ** 24)
    if not 0 <= U < 2 ** 24:
        raise ValueError("u_resample must lie in [0, 1)")
    if sum(R) == 0:
        Pw = [int(v) for v in np.floor(p_row.astype(np.float64) * 2.0 ** 40)]
        if sum(Pw) == 0:
            raise ValueError("target row has no mass")
        return _draw(Pw, U)
    return _draw(R, U)


def rejection(p: np.ndarray, q: np.ndarray, draft: np.ndarray,
              u_accept: np.ndarray, u_resample: np.ndarray):
    """Speculative rejection sampling over a block.

    p, q [S, K, V] float32 probabilities; draft [S, K]; u_accept [S, K] and
    u_resample [S] float32 uniforms in [0, 1).  Returns accept_len [S] and
    next_token [S] (resampled token at row accept_len, -1 if all accepted).
    """
    S, K, _ = p.shape
    acc = np.zeros(S, dtype=np.int32)
    nxt = np.full(S, -1, dtype=np.int32)
    for s in range(S):
        a = K
        for i in range(K):
            x = int(draft[s, i])
            if not float(u_accept[s, i]) * float(q[s, i, x]) < float(p[s, i, x]):
                a = i
                break
        acc[s] = a
        if a < K:
            nxt[s] = residual_sample(p[s, a], q[s, a], u_resample[s])
    return acc, nxt


def greedy_bonus(logits: np.ndarray, draft: np.ndarray):
    """Greedy acceptance with a bonus row.  logits [S, K+1, V], draft [S, K].

    Rows 0..K-1 check drafts 0..K-1 as in `greedy`; row K is the target's
    prediction after the whole block.  Returns accept_len [S] in [0, K] and
    next_token [S] = argmax of row accept_len (the bonus row when all K drafts
    were accepted), never -1.
    """
    S, K1, _ = logits.shape
    K = K1 - 1
    if draft.shape != (S, K):
        raise ValueError("draft must be [S, K] for logits [S, K+1, V]")
    acc = np.zeros(S, dtype=np.int32)
    nxt = np.zeros(S, dtype=np.int32)
    for s in range(S):
        a = K
        for i in range(K):
            if argmax_lowest(logits[s, i]) != int(draft[s, i]):
                a = i
                break
        acc[s] = a
        nxt[s] = argmax_lowest(logits[s, a])
    return acc, nxt


def bonus_sample(p_row: np.ndarray, u_resample: float) -> int:
    """Token drawn from the target row p by the integer inverse-CDF rule."""
    Pw = [int(v) for v in np.floor(p_row.astype(np.float64) * 2.0 ** 40)]
    U = int(float(u_resample) * 2 ** 24)
    if not 0 <= U < 2 ** 24:
        raise ValueError("u_resample must lie in [0, 1)")
    if sum(Pw) == 0:
        raise ValueError("target row has no mass")
    return _draw(Pw, U)


def rejection_bonus(p: np.ndarray, q: np.ndarray, draft: np.ndarray,
                    u_accept: np.ndarray, u_resample: np.ndarray):
    """Rejection sampling with a bonus row.  p [S, K+1, V] (row K: the target
    after the block), q [S, K, V], draft [S, K], u_accept [S, K], u_resample
    [S].  As `rejection` on rows 0..K-1; when all K drafts are accepted the
    next token is drawn from p[s, K] (`bonus_sample`) instead of -1."""
    S, K1, _ = p.shape
    K = K1 - 1
    if q.shape[:2] != (S, K) or draft.shape != (S, K):
        raise ValueError("q [S, K, V] and draft [S, K] for p [S, K+1, V]")
    acc, nxt = rejection(p[:, :K], q, draft, u_accept, u_resample)
    for s in range(S):
        if acc[s] == K:
            nxt[s] = bonus_sample(p[s, K], u_resample[s])
    return acc, nxt

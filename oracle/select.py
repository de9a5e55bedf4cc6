"""KVMem-style block summaries, block scores and top-k selection -- CPU oracle.

Test infrastructure only.

The KVMem reproduction (lcz.me/topic/1972; test command and recall sections)
keeps, per request, a GPU working set made of 128-token blocks: the blocks a
retrieval query ranks highest fill a token budget (32,768 tokens = 256 blocks),
and the most recent tokens (a 16,384-token reserve = 128 blocks) are always kept.
The pages do not say how a block is ranked.  The reading used here (the plainest
one the workload definitions support):

* summary[b]  = mean over the block's 128 tokens of the dequantised key, per
                channel, rounded once to fp32;
* score[b]    = sum over the KV head's query-head group j and channels c of
                q[j][c] * summary[b][c], rounded once to float64 (the fp32 x fp32
                products are exact in float64; math.fsum rounds the sum once);
* selection   = the `budget` highest-scoring blocks among the full blocks older
                than the recent window (ties: lower block index first), united
                with the recent window and any partial tail blocks, in ascending
                logical order.
"""
from __future__ import annotations

import math

import numpy as np


def _grid(v: np.ndarray) -> np.ndarray:
    """Spacing of the float16 grid at |v| (11 significant bits), inf where v == 0; smaller
    than the true spacing for fp16 subnormals, which only makes the check stricter."""
    _, e = np.frexp(np.where(v == 0, 1.0, v))
    return np.where(v == 0, np.inf, np.ldexp(1.0, e - 11))


def block_summaries(codes: np.ndarray, d: np.ndarray, fmt: str = "q8_0") -> np.ndarray:
    """Mean dequantised key of each block, keys stored as Q8_0, Q4_0, Q5_0 or Q5_1.

    codes: [n_blocks][128][8][32] (int8 for Q8_0, 0..15 for Q4_0, 0..31 for Q5_0 / Q5_1);
    d: float16 [n_blocks][128][8] ([n_blocks][128][8][2] = (d, m) for Q5_1).  Returns fp32
    [n_blocks][256].  The key value is q * d for Q8_0, (q - 8) * d for Q4_0, (q - 16) * d
    for Q5_0 and q * d + m for Q5_1.

    Each product d * q is exact in float64 (11 + 8 significant bits) and, like each
    minimum m, a multiple of the block's smallest fp16 grid step; when the sum of
    magnitudes stays below 2**53 grid steps every partial sum is exact, so the float64 sum
    below is the exact sum (checked, not assumed).  Division by 128 is exact; the one
    rounding is the final conversion to fp32.
    """
    if fmt not in ("q8_0", "q4_0", "q5_0", "q5_1"):
        raise ValueError(f"unsupported key format {fmt}")
    codes = np.asarray(codes)
    nb = codes.shape[0]
    dd = np.asarray(d, dtype=np.float16).astype(np.float64)
    d64 = dd[..., 0] if fmt == "q5_1" else dd                         # [nb][128][8]
    q = codes.astype(np.float64) - {"q4_0": 8.0, "q5_0": 16.0}.get(fmt, 0.0)
    terms = [q * d64[..., None]]                                      # [nb][128][8][32]
    grids = [_grid(d64)]
    if fmt == "q5_1":
        m64 = dd[..., 1]
        terms.append(np.broadcast_to(m64[..., None], q.shape))
        grids.append(_grid(m64))
    # exactness certificate
    grid = np.minimum.reduce([g.reshape(nb, -1).min(axis=1) for g in grids])
    mag = sum(np.abs(t).reshape(nb, -1).sum(axis=1) for t in terms)
    if np.any(np.isfinite(grid) & (mag >= np.ldexp(grid, 53))):
        raise ArithmeticError("block sum not exactly representable in float64")
    s = sum(t.sum(axis=1) for t in terms)                            # [nb][8][32] exact
    return (s / 128.0).reshape(nb, -1).astype(np.float32)


def block_scores(summaries: np.ndarray, q_group: np.ndarray) -> np.ndarray:
    """summaries fp32 [n_blocks][256]; q_group fp32 [g][256] -> float64 [n_blocks]."""
    S = np.asarray(summaries, dtype=np.float32).astype(np.float64)
    Q = np.asarray(q_group, dtype=np.float32).astype(np.float64)
    out = np.empty(S.shape[0])
    for b in range(S.shape[0]):
        out[b] = math.fsum((Q * S[b][None, :]).ravel())
    return out


def select_blocks(scores: np.ndarray, n_full: int, n_total: int, budget: int, recent: int):
    """Top-`budget` candidates plus the recent window and partial tail blocks.

    scores: float64 [>= n_full] (only [0, n_full - recent) are read).
    Returns (ascending int32 logical block ids, cut gap).  The cut gap is the
    score difference between the last selected and the first rejected candidate
    (inf when nothing is rejected): a small gap makes the selection fragile
    under any rounding difference, so tests reject such seeds."""
    recent = max(0, min(recent, n_full))
    n_cand = n_full - recent
    cand = np.arange(n_cand)
    order = sorted(cand.tolist(), key=lambda b: (-scores[b], b))
    take = order[:budget]
    gap = math.inf
    if len(order) > budget and budget > 0:
        gap = scores[order[budget - 1]] - scores[order[budget]]
    sel = sorted(set(take) | set(range(n_cand, n_total)))
    return np.asarray(sel, dtype=np.int32), gap

"""Masked softmax attention with log-sum-exp, and the LSE merge -- CPU oracle.

Test infrastructure only.

What the path computes (Adaptive KV Streaming + RDNA 4 announcement, wqu.guru,
method list: paged decode attention extended to verify batches; chunked prefill
across streamed pages merged by online log-sum-exp):

    s[r, t]  = (q[r] . k[t]) * scale            for key positions pos[t] <= qpos[r]
    m[r]     = max_t s[r, t]
    l[r]     = sum_t exp(s[r, t] - m[r])
    o[r]     = sum_t exp(s[r, t] - m[r]) * v[t] / l[r]
    lse[r]   = m[r] + ln l[r]                                   (natural log)

A row with no visible key gives o = 0 and lse = -inf (a reading: the pages never
reach that case).  ``scale`` is 1/sqrt(head_dim) = 1/16 for head_dim 256.

The merge of partial results (o_i, lse_i) over disjoint key sets is

    lse = ln sum_i exp(lse_i),     o = sum_i exp(lse_i - lse) * o_i,

skipping parts with lse_i = -inf; it reproduces single-pass attention exactly in
exact arithmetic, which the tests check.
"""
from __future__ import annotations

import numpy as np


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, key_pos, q_pos, scale: float):
    """q: [R][D]; k, v: [T][D] (dequantised); key_pos [T]; q_pos [R].

    Returns (o [R][D] float64, lse [R] float64)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    key_pos = np.asarray(key_pos, dtype=np.int64)
    q_pos = np.asarray(q_pos, dtype=np.int64)
    R, D = q.shape
    if k.shape[0] == 0:
        return np.zeros((R, v.shape[1] if v.ndim == 2 else D)), np.full(R, -np.inf)
    s = (q @ k.T) * float(scale)
    visible = key_pos[None, :] <= q_pos[:, None]
    s = np.where(visible, s, -np.inf)
    m = np.max(s, axis=1)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    p = np.where(visible, np.exp(s - m_safe[:, None]), 0.0)
    l = p.sum(axis=1)
    o = np.zeros((R, v.shape[1]))
    ok = ~empty
    o[ok] = (p[ok] @ v) / l[ok, None]
    lse = np.full(R, -np.inf)
    lse[ok] = m[ok] + np.log(l[ok])
    return o, lse


def merge_lse(o_parts: np.ndarray, lse_parts: np.ndarray):
    """o_parts [P][R][D], lse_parts [P][R] -> (o [R][D], lse [R]), float64."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    P, R = lse_parts.shape
    mx = np.max(lse_parts, axis=0)
    empty = ~np.isfinite(mx)
    mx_safe = np.where(empty, 0.0, mx)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - mx_safe[None, :]), 0.0)
    tot = w.sum(axis=0)
    lse = np.full(R, -np.inf)
    lse[~empty] = mx[~empty] + np.log(tot[~empty])
    o = np.zeros(o_parts.shape[1:])
    ok = ~empty
    o[ok] = np.einsum("pr,prd->rd", w[:, ok] / tot[None, ok], o_parts[:, ok])
    return o, lse


def attend_chunked(q, k, v, key_pos, q_pos, scale, chunk: int):
    """Attention over key chunks of `chunk` keys, merged by merge_lse."""
    T = np.asarray(k).shape[0]
    parts_o, parts_l = [], []
    for a in range(0, max(T, 1), chunk):
        o, l = attend(q, np.asarray(k)[a:a + chunk], np.asarray(v)[a:a + chunk],
                      np.asarray(key_pos)[a:a + chunk], q_pos, scale)
        parts_o.append(o)
        parts_l.append(l)
    return merge_lse(np.stack(parts_o), np.stack(parts_l))


def gather_pages(codes_pages, d_pages, fmt: str, page_ids, logical_ids, page_tokens: int = 128):
    """Dequantise the listed pages into (k or v [T][D] float64, key positions [T]).

    codes_pages: [n_phys][128][8][32]; d_pages: [n_phys][128][8] (fp16);
    page_ids: physical ids in list order; logical_ids: their logical block indices."""
    from .quant import dequantize

    page_ids = np.asarray(page_ids, dtype=np.int64)
    logical_ids = np.asarray(logical_ids, dtype=np.int64)
    x = dequantize(codes_pages[page_ids], d_pages[page_ids], fmt)  # [n][128][256]
    pos = (logical_ids[:, None] * page_tokens + np.arange(page_tokens)[None, :]).reshape(-1)
    return x.reshape(-1, x.shape[-1]), pos

"""Hadamard-rotated KV -- CPU oracle.

Test infrastructure only.

The Vulkan speculative-decoding report, 7900 XTX (lcz.me/topic/1398), in its pitfalls
section (the item on attention rotation), runs q8_0 / q5_1 / q4_0 KV caches with the
attention rotation on and notes that the rotation improves the precision of the quantized KV.  The page does not write the transform out; the
reading used here (the plainest one, and the one that keeps attention unchanged in exact
arithmetic):

* R = H / 16 with H the 256 x 256 Sylvester-Hadamard matrix (H[i][j] = (-1)^popcount(i & j));
  R is symmetric and orthonormal, so R R = I;
* keys and values of every head are rotated before quantization (k' = k R, v' = v R) and the
  query is rotated the same way (q' = q R), so q' . k' = q . k;
* the attention output over the rotated values is rotated back: o = o' R.
"""
from __future__ import annotations

import numpy as np

from oracle import attention as oatt
from oracle import quant as oq


def hadamard_matrix(n: int = 256) -> np.ndarray:
    """Sylvester construction H_n (entries +-1), n a power of two."""
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def rotation(n: int = 256) -> np.ndarray:
    """The orthonormal rotation R = H_n / sqrt(n)."""
    return hadamard_matrix(n) / np.sqrt(n)


def rotate(x: np.ndarray) -> np.ndarray:
    """x R over the last axis (float64)."""
    return np.asarray(x, np.float64) @ rotation(np.shape(x)[-1])


def attend_quantized(q, k, v, k_pos, q_pos, v_fmt="q4_0", rotated=False):
    """Attention of query rows q [rows][256] over keys/values k, v [T][256] (fp32) stored as
    Q8_0 K and v_fmt V, optionally through the rotation.  Returns (o, lse) in float64."""
    if rotated:
        q = rotate(q)
        k = rotate(k).astype(np.float32)
        v = rotate(v).astype(np.float32)
    kc, kd = oq.q8_0_quantize(np.asarray(k, np.float32))
    vc, vd = oq.quantize(np.asarray(v, np.float32), v_fmt)
    kh = oq.q8_0_dequantize(kc, kd)
    vh = oq.dequantize(vc, vd, v_fmt)
    o, lse = oatt.attend(np.asarray(q, np.float64), kh, vh, k_pos, q_pos, 1.0 / 16.0)
    if rotated:
        o = rotate(o)
    return o, lse

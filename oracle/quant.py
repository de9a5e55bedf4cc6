"""Q8_0, Q4_0, Q5_0, Q4_1 and Q5_1 block quantisation -- CPU oracle (test infrastructure only).

Both formats split a row into blocks of 32 elements and store one fp16 scale
``d`` per block (Vulkan speculative-decoding report, lcz.me/topic/1398, section
"pitfalls": legacy block quants only; q8_0 = 8.5 bits per element, i.e. 32 int8 +
fp16 = 34 bytes per block; q4_0 K+V = 18 KiB per token, i.e. 16 bytes of nibbles
+ fp16 = 18 bytes per block).

The pages do not spell out the encoders.  The readings used here:

* Q8_0: ``d = amax / 127`` in fp32, ``q = round_half_away(x * (1/d))`` with the
  reciprocal and the product each rounded to fp32, clamped to [-127, 127]; the
  stored scale is fp16(d) (round to nearest even).  ``amax == 0`` gives d = 0 and
  q = 0.  Value = q * d_fp16.
* Q4_0: value = (q - 8) * d with q in [0, 15].  ``m`` = the signed element of
  largest magnitude (first one on ties), ``d = m / -8`` in fp32, ``q =
  min(15, floor(x * (1/d) + 8.5))`` with the product and the sum each rounded to
  fp32; the element m maps to q = 0.  ``m == 0`` gives d = 0 and q = 8.

* Q5_1 (section "pitfalls" of the same report: a 5-bit format with a zero point,
  6 bits per element, i.e. 32 x 5 bits + fp16 scale + fp16 minimum = 24 bytes per
  block; the report pairs Q5_1 keys with Q4_0 values): value = q * d + m with q in
  [0, 31].  ``m`` = the block minimum, ``d = (max - min) / 31`` (the difference and the
  quotient each rounded to fp32), ``q = min(31, floor((x - m) * (1/d) + 0.5))`` with the
  difference, the product and the sum each rounded to fp32; d and m are stored as fp16.
  ``max == min`` gives d = 0 and q = 0.  The scale pair is carried as one float16 array
  [..., n, 2] holding (d, m).

* Q5_0 and Q4_1 (named with Q5_1 in the same section's list of KV formats; the MTP tuning
  notes on one 7900 XTX, lcz.me/topic/593, run a Q5_0 K / Q4_1 V cache at 128K): Q5_0 is
  Q4_0 with 5-bit codes, value = (q - 16) * d, ``d = m / -16``, ``q = min(31, floor(x *
  (1/d) + 16.5))`` (22 bytes per block); Q4_1 is Q5_1 with 4-bit codes, value = q * d + m,
  ``d = (max - min) / 15``, ``q = min(15, floor((x - m) * (1/d) + 0.5))`` (20 bytes per
  block).  Same rounding rules as Q4_0 and Q5_1.

Every rounding that decides an integer code is done in fp32, exactly as an IEEE
fp32 unit would do it, so a GPU encoder can match the codes bit for bit.
"""
from __future__ import annotations

import numpy as np

QK = 32  # elements per block

F32 = np.float32


def _blocks(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=F32)
    if x.shape[-1] % QK:
        raise ValueError("last axis must be a multiple of 32")
    return x.reshape(x.shape[:-1] + (x.shape[-1] // QK, QK))


def _recip_f32(d: np.ndarray) -> np.ndarray:
    """1/d rounded to fp32, and 0 where d == 0.

    A nonzero fp32 scale whose reciprocal overflows (|d| below about 2.9e-39: a block whose
    elements, or whose spread for the zero-point formats, are all below about 1e-36) has no
    defined codes under these readings; such blocks are outside the supported input range and
    are refused."""
    out = np.zeros_like(d, dtype=F32)
    nz = d != 0
    with np.errstate(over="ignore"):
        out[nz] = F32(1.0) / d[nz]
    if not np.all(np.isfinite(out)):
        raise ValueError("block scale so small that 1/d overflows fp32: outside the supported input range")
    return out


def round_half_away(y: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest integer, halves away from zero (exact)."""
    y64 = np.asarray(y, dtype=np.float64)  # exact widening
    return np.sign(y64) * np.floor(np.abs(y64) + 0.5)


def q8_0_quantize(x: np.ndarray):
    """x: fp32 [..., 32n] -> (qs int8 [..., n, 32], d float16 [..., n])."""
    xb = _blocks(x)
    amax = np.max(np.abs(xb), axis=-1)
    d32 = (amax / F32(127.0)).astype(F32)
    inv = _recip_f32(d32)
    y = (xb * inv[..., None]).astype(F32)
    q = np.clip(round_half_away(y), -127, 127)
    return q.astype(np.int8), d32.astype(np.float16)


def q8_0_dequantize(qs: np.ndarray, d: np.ndarray) -> np.ndarray:
    """(qs [..., n, 32], d [..., n]) -> float64 [..., 32n], value = q * d."""
    v = qs.astype(np.float64) * d.astype(np.float64)[..., None]
    return v.reshape(v.shape[:-2] + (-1,))


def _offset_quantize(x: np.ndarray, half: int):
    """Symmetric codes with offset `half` (8 for Q4_0, 16 for Q5_0): m = the signed element of
    largest magnitude (first on ties), d = m / -half, q = min(2 half - 1, floor(x/d + half + .5))."""
    xb = _blocks(x)
    idx = np.argmax(np.abs(xb), axis=-1)
    m = np.take_along_axis(xb, idx[..., None], axis=-1)[..., 0]
    d32 = (m / F32(-half)).astype(F32)
    inv = _recip_f32(d32)
    y = (xb * inv[..., None]).astype(F32)
    z = (y + F32(half + 0.5)).astype(F32)
    q = np.minimum(2 * half - 1, np.floor(z.astype(np.float64)))
    return q.astype(np.uint8), d32.astype(np.float16)


def _min_quantize(x: np.ndarray, top: int):
    """Codes with a zero point (top = 15 for Q4_1, 31 for Q5_1): m = the block minimum,
    d = (max - m) / top, q = min(top, floor((x - m)/d + 0.5)); returns (q, (d, m))."""
    xb = _blocks(x)
    mn = np.min(xb, axis=-1)
    mx = np.max(xb, axis=-1)
    d32 = ((mx - mn).astype(F32) / F32(top)).astype(F32)
    inv = _recip_f32(d32)
    y = ((xb - mn[..., None]).astype(F32) * inv[..., None]).astype(F32)
    z = (y + F32(0.5)).astype(F32)
    q = np.minimum(top, np.floor(z.astype(np.float64)))
    dm = np.stack([d32.astype(np.float16), mn.astype(np.float16)], axis=-1)
    return q.astype(np.uint8), dm


def q4_0_quantize(x: np.ndarray):
    """x: fp32 [..., 32n] -> (q uint8 in [0,15] [..., n, 32], d float16 [..., n])."""
    return _offset_quantize(x, 8)


def q4_0_dequantize(q: np.ndarray, d: np.ndarray) -> np.ndarray:
    """(q [..., n, 32], d [..., n]) -> float64 [..., 32n], value = (q - 8) * d."""
    v = (q.astype(np.float64) - 8.0) * d.astype(np.float64)[..., None]
    return v.reshape(v.shape[:-2] + (-1,))


def q5_0_quantize(x: np.ndarray):
    """x: fp32 [..., 32n] -> (q uint8 in [0,31] [..., n, 32], d float16 [..., n])."""
    return _offset_quantize(x, 16)


def q5_0_dequantize(q: np.ndarray, d: np.ndarray) -> np.ndarray:
    """(q [..., n, 32], d [..., n]) -> float64 [..., 32n], value = (q - 16) * d."""
    v = (q.astype(np.float64) - 16.0) * d.astype(np.float64)[..., None]
    return v.reshape(v.shape[:-2] + (-1,))


def q5_1_quantize(x: np.ndarray):
    """x: fp32 [..., 32n] -> (q uint8 in [0,31] [..., n, 32], (d, m) float16 [..., n, 2])."""
    return _min_quantize(x, 31)


def q4_1_quantize(x: np.ndarray):
    """x: fp32 [..., 32n] -> (q uint8 in [0,15] [..., n, 32], (d, m) float16 [..., n, 2])."""
    return _min_quantize(x, 15)


def min_dequantize(q: np.ndarray, dm: np.ndarray) -> np.ndarray:
    """Q4_1 / Q5_1: (q [..., n, 32], (d, m) [..., n, 2]) -> float64 [..., 32n], value = q * d + m."""
    dm = np.asarray(dm, dtype=np.float16).astype(np.float64)
    v = q.astype(np.float64) * dm[..., 0][..., None] + dm[..., 1][..., None]
    return v.reshape(v.shape[:-2] + (-1,))


q5_1_dequantize = min_dequantize
q4_1_dequantize = min_dequantize

_QUANT = {"q8_0": q8_0_quantize, "q4_0": q4_0_quantize, "q5_0": q5_0_quantize, "q4_1": q4_1_quantize,
          "q5_1": q5_1_quantize}
_DEQUANT = {"q8_0": q8_0_dequantize, "q4_0": q4_0_dequantize, "q5_0": q5_0_dequantize,
            "q4_1": min_dequantize, "q5_1": min_dequantize}


def quantize(x: np.ndarray, fmt: str):
    return _QUANT[fmt](x)


def dequantize(codes: np.ndarray, d: np.ndarray, fmt: str) -> np.ndarray:
    return _DEQUANT[fmt](codes, d)


def block_bytes(fmt: str) -> int:
    """Bytes of one 32-element block: fp16 scale (and fp16 minimum) + codes."""
    return {"q8_0": 2 + 32, "q4_0": 2 + 16, "q5_0": 2 + 20, "q4_1": 2 + 2 + 16, "q5_1": 2 + 2 + 20}[fmt]

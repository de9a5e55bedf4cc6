"""Byte layout of one 128-token KV page -- CPU oracle (test infrastructure only).

A page holds the K (or V) rows of 128 consecutive tokens of one (layer, KV head)
(KVMem reproduction, lcz.me/topic/1972, test command: 128-token blocks).  The
pages fix only the bits per element; the arrangement below is this library's own
storage spec, written so that one 16-byte load per thread feeds tensor-core
fragments directly.  Bytes per page equal the AoS block sizes the pages print:
K Q8_0 = 128 x 8 x 34 = 34,816; K Q4_0 = V Q4_0 = 128 x 8 x 18 = 18,432; K Q5_1 = 128 x 8 x 24
= 24,576; K Q5_0 = 128 x 8 x 22 = 22,528; V Q4_1 = 128 x 8 x 20 = 20,480; V Q8_0 = 34,816.

Notation: tok in [0,128) is the token slot inside the page, dim in [0,256) the
channel, b = dim // 32 the block, d[tok][b] the fp16 block scale.  Tokens are
grouped in sixteens: G = tok // 16.

K page, Q8_0 (34,816 bytes)
  codes, bytes [0, 32768): byte at
      ((((G*4 + P)*2 + H)*8 + R)*4 + T)*16 + j          (P<4, H<2, R<8, T<4, j<16)
  holds the code q (in [-127, 127]) of token 16G + 8H + R, channel
  64P + 32*(j // 8) + 8T + (j % 8), stored offset-binary as the byte q + 128 (the value of the
  byte XOR 0x80 read as int8; a zero byte is the code -128, so an unwritten slot, whose
  scale is zero too, holds the value 0).
  scales, bytes [32768, 34816): fp16 at 32768 + 2*((((G*8 + R)*2 + H)*8) + b)
  holds d[16G + 8H + R][b].

K page, Q4_0 (18,432 bytes)
  nibbles, bytes [0, 16384): the little-endian 32-bit word at byte
      4 * (((((G*2 + Q)*2 + H)*8 + R)*4 + T)*4 + c)       (Q<2, H<2, R<8, T<4, c<4)
  belongs to token 16G + 8H + R and block b = 4Q + c; it holds the 4-bit codes of the
  channels 32b + 8T + i (i < 8), channel i at bit 4*(i // 2) + 16*(i % 2).
  scales, bytes [16384, 18432): same arrangement as the Q8_0 K scales.

K page, Q5_1 (24,576 bytes)
  low nibbles, bytes [0, 16384): the low 4 bits of every code, arranged as the K Q4_0 nibbles.
  fifth bits, bytes [16384, 20480): the little-endian 32-bit word at byte
      16384 + 4 * ((((G*2 + Q)*2 + H)*8 + R)*4 + T)
  holds bit 4 of the codes of token 16G + 8H + R, channels 32(4Q + c) + 8T + i (c < 4, i < 8),
  channel (c, i) at bit 16*(i % 2) + 4c + i // 2.
  scales d, bytes [20480, 22528), and minima m, bytes [22528, 24576): fp16 at base + 2*idx
  with idx the K Q8_0 scale index ((G*8 + R)*2 + H)*8 + b.  The value is q * d + m.

K page, Q5_0 (22,528 bytes)
  low nibbles and fifth bits as the K Q5_1 page, bytes [0, 20480); scales d, bytes
  [20480, 22528), as the K Q5_1 scales.  The value is (q - 16) * d.

V page, Q4_0 (18,432 bytes)
  nibbles, bytes [0, 16384): byte at
      ((((G*4 + C)*8 + R)*4 + T)*16 + 4*w + y            (C<4, R<8, T<4, w<4, y<4)
  belongs to block b = 2C + w // 2 and token 16G + 2T + 8*(w % 2) + y // 2; its
  low nibble is channel 32b + 16*(y % 2) + R and its high nibble that channel + 8.
  A nibble stores q in [0, 15]; the value is (q - 8) * d.
  scales, bytes [16384, 18432): fp16 at 16384 + 2*((((G*4 + T)*8 + b)*4) + k)
  holds d[16G + 2T + (k % 2) + 8*(k // 2)][b]                (k < 4).

V page, Q4_1 (20,480 bytes)
  nibbles, bytes [0, 16384), and scales d, bytes [16384, 18432), as the V Q4_0 page; minima m,
  bytes [18432, 20480), in the arrangement of the scales.  The value is q * d + m.

V page, Q8_0 (34,816 bytes)
  codes, bytes [0, 32768): byte at
      ((((G*8 + b)*8 + R)*4 + T)*16 + 4*w + y            (b<8, R<8, T<4, w<4, y<4)
  holds the code of token 16G + 2T + 8*(w % 2) + y % 2, channel
  32b + 16*(w // 2) + 8*(y // 2) + R, offset-binary as for the K Q8_0 codes.
  scales, bytes [32768, 34816): same arrangement as the Q4_0 V scales.
"""
from __future__ import annotations

import numpy as np

PAGE_TOKENS = 128
HEAD_DIM = 256
N_BLOCKS = HEAD_DIM // 32

K_Q8_BYTES = 34816
K_Q4_BYTES = 18432
K_Q51_BYTES = 24576
K_Q50_BYTES = 22528
V_Q41_BYTES = 20480
V_Q4_BYTES = 18432
V_Q8_BYTES = 34816


def page_bytes(role: str, fmt: str) -> int:
    if role == "k" and fmt == "q8_0":
        return K_Q8_BYTES
    if role == "k" and fmt == "q4_0":
        return K_Q4_BYTES
    if role == "k" and fmt == "q5_1":
        return K_Q51_BYTES
    if role == "k" and fmt == "q5_0":
        return K_Q50_BYTES
    if role == "v" and fmt == "q4_1":
        return V_Q41_BYTES
    if role == "v" and fmt == "q4_0":
        return V_Q4_BYTES
    if role == "v" and fmt == "q8_0":
        return V_Q8_BYTES
    raise ValueError(f"unsupported page kind {role}/{fmt}")


def _k_code_map():
    G, P, H, R, T, j = np.meshgrid(np.arange(8), np.arange(4), np.arange(2), np.arange(8),
                                   np.arange(4), np.arange(16), indexing="ij")
    off = ((((G * 4 + P) * 2 + H) * 8 + R) * 4 + T) * 16 + j
    tok = 16 * G + 8 * H + R
    dim = 64 * P + 32 * (j // 8) + 8 * T + (j % 8)
    return off.ravel(), tok.ravel(), dim.ravel()


def _k_scale_map():
    G, R, H, b = np.meshgrid(np.arange(8), np.arange(8), np.arange(2), np.arange(8), indexing="ij")
    idx = ((G * 8 + R) * 2 + H) * 8 + b
    return idx.ravel(), (16 * G + 8 * H + R).ravel(), b.ravel()


def _v_scale_map():
    G, T, b, k = np.meshgrid(np.arange(8), np.arange(4), np.arange(8), np.arange(4), indexing="ij")
    idx = ((G * 4 + T) * 8 + b) * 4 + k
    tok = 16 * G + 2 * T + (k % 2) + 8 * (k // 2)
    return idx.ravel(), tok.ravel(), b.ravel()


def _v4_nibble_map():
    G, C, R, T, w, y = np.meshgrid(np.arange(8), np.arange(4), np.arange(8), np.arange(4),
                                   np.arange(4), np.arange(4), indexing="ij")
    off = ((((G * 4 + C) * 8 + R) * 4 + T) * 16) + 4 * w + y
    b = 2 * C + w // 2
    tok = 16 * G + 2 * T + 8 * (w % 2) + y // 2
    lo = 32 * b + 16 * (y % 2) + R
    return off.ravel(), tok.ravel(), lo.ravel(), (lo + 8).ravel()


def _k4_nibble_map():
    """(byte offset, shift, token, channel) of every K Q4_0 code."""
    G, Q, H, R, T, c, i = np.meshgrid(np.arange(8), np.arange(2), np.arange(2), np.arange(8),
                                      np.arange(4), np.arange(4), np.arange(8), indexing="ij")
    word = ((((G * 2 + Q) * 2 + H) * 8 + R) * 4 + T) * 4 + c
    bit = 4 * (i // 2) + 16 * (i % 2)
    off = 4 * word + bit // 8
    tok = 16 * G + 8 * H + R
    dim = 32 * (4 * Q + c) + 8 * T + i
    return off.ravel(), (bit % 8).ravel(), tok.ravel(), dim.ravel()


def _k5_high_bit_map():
    """(byte offset, bit in byte, token, channel) of bit 4 of every K Q5_1 code."""
    G, Q, H, R, T, c, i = np.meshgrid(np.arange(8), np.arange(2), np.arange(2), np.arange(8),
                                      np.arange(4), np.arange(4), np.arange(8), indexing="ij")
    word = (((G * 2 + Q) * 2 + H) * 8 + R) * 4 + T
    bit = 16 * (i % 2) + 4 * c + i // 2
    off = 16384 + 4 * word + bit // 8
    tok = 16 * G + 8 * H + R
    dim = 32 * (4 * Q + c) + 8 * T + i
    return off.ravel(), (bit % 8).ravel(), tok.ravel(), dim.ravel()


def _v8_code_map():
    G, b, R, T, w, y = np.meshgrid(np.arange(8), np.arange(8), np.arange(8), np.arange(4),
                                   np.arange(4), np.arange(4), indexing="ij")
    off = ((((G * 8 + b) * 8 + R) * 4 + T) * 16) + 4 * w + y
    tok = 16 * G + 2 * T + 8 * (w % 2) + y % 2
    dim = 32 * b + 16 * (w // 2) + 8 * (y // 2) + R
    return off.ravel(), tok.ravel(), dim.ravel()


_K_CODES = _k_code_map()
_K_SCALES = _k_scale_map()
_V_SCALES = _v_scale_map()
_V4_NIBBLES = _v4_nibble_map()
_V8_CODES = _v8_code_map()
_K4_NIBBLES = _k4_nibble_map()
_K5_HIGH = _k5_high_bit_map()


def _flat_codes(codes: np.ndarray) -> np.ndarray:
    """[128][8][32] block codes -> [128][256] channel codes."""
    return np.asarray(codes).reshape(PAGE_TOKENS, HEAD_DIM)


def _offset_binary(q: np.ndarray) -> np.ndarray:
    """Q8_0 codes in [-128, 127] -> their stored bytes q + 128."""
    q = np.asarray(q).astype(np.int16)
    if np.any(q < -128) or np.any(q > 127):
        raise ValueError("Q8_0 codes must be in [-128, 127]")
    return (q + 128).astype(np.uint8)


def encode_page(role: str, fmt: str, codes: np.ndarray, d: np.ndarray) -> np.ndarray:
    """Encode one page.  codes: [128][8][32] (int8 for Q8_0, 0..15 for Q4_0 / Q4_1, 0..31 for
    Q5_0 / Q5_1); d: [128][8] float16 ([128][8][2] (d, m) for Q4_1 and Q5_1).  Returns
    uint8[page_bytes]."""
    n = page_bytes(role, fmt)
    out = np.zeros(n, dtype=np.uint8)
    c = _flat_codes(codes)
    d16 = np.asarray(d, dtype=np.float16).view(np.uint16)
    if role == "k" and fmt in ("q5_1", "q5_0"):
        c8 = c.astype(np.uint8)
        if np.any(c8 > 31):
            raise ValueError("5-bit codes must be in [0, 31]")
        off, sh, tok, dim = _K4_NIBBLES
        np.bitwise_or.at(out, off, ((c8[tok, dim] & 15) << sh).astype(np.uint8))
        off, sh, tok, dim = _K5_HIGH
        np.bitwise_or.at(out, off, ((c8[tok, dim] >> 4) << sh).astype(np.uint8))
        idx, tok, b = _K_SCALES
        parts = ((20480, d16[..., 0]), (22528, d16[..., 1])) if fmt == "q5_1" else ((20480, d16),)
        for base, part in parts:
            sv = part[tok, b]
            out[base + 2 * idx] = (sv & 0xFF).astype(np.uint8)
            out[base + 2 * idx + 1] = (sv >> 8).astype(np.uint8)
        return out
    if role == "v" and fmt == "q4_1":
        off, tok, lo, hi = _V4_NIBBLES
        c8 = c.astype(np.uint8)
        if np.any(c8 > 15):
            raise ValueError("Q4_1 codes must be in [0, 15]")
        out[off] = c8[tok, lo] | (c8[tok, hi] << 4)
        idx, tok, b = _V_SCALES
        for base, part in ((16384, d16[..., 0]), (18432, d16[..., 1])):
            sv = part[tok, b]
            out[base + 2 * idx] = (sv & 0xFF).astype(np.uint8)
            out[base + 2 * idx + 1] = (sv >> 8).astype(np.uint8)
        return out
    if role == "k" and fmt == "q4_0":
        off, sh, tok, dim = _K4_NIBBLES
        c8 = c.astype(np.uint8)
        if np.any(c8 > 15):
            raise ValueError("Q4_0 codes must be in [0, 15]")
        np.bitwise_or.at(out, off, (c8[tok, dim] << sh).astype(np.uint8))
        idx, tok, b = _K_SCALES
        scale_base = 16384
    elif role == "k":
        off, tok, dim = _K_CODES
        out[off] = _offset_binary(c[tok, dim])
        idx, tok, b = _K_SCALES
        scale_base = 32768
    elif fmt == "q4_0":
        off, tok, lo, hi = _V4_NIBBLES
        c8 = c.astype(np.uint8)
        if np.any(c8 > 15):
            raise ValueError("Q4_0 codes must be in [0, 15]")
        out[off] = c8[tok, lo] | (c8[tok, hi] << 4)
        idx, tok, b = _V_SCALES
        scale_base = 16384
    else:
        off, tok, dim = _V8_CODES
        out[off] = _offset_binary(c[tok, dim])
        idx, tok, b = _V_SCALES
        scale_base = 32768
    sv = d16[tok, b]
    out[scale_base + 2 * idx] = (sv & 0xFF).astype(np.uint8)
    out[scale_base + 2 * idx + 1] = (sv >> 8).astype(np.uint8)
    return out


def decode_page(role: str, fmt: str, page: np.ndarray):
    """Inverse of encode_page: uint8[page_bytes] -> (codes [128][8][32], d [128][8] f16)."""
    page = np.asarray(page, dtype=np.uint8)
    if page.size != page_bytes(role, fmt):
        raise ValueError("wrong page size")
    c = np.zeros((PAGE_TOKENS, HEAD_DIM), dtype=np.int16)
    if role == "k" and fmt in ("q5_1", "q5_0"):
        off, sh, tok, dim = _K4_NIBBLES
        c[tok, dim] = (page[off] >> sh) & 0xF
        off, sh, tok, dim = _K5_HIGH
        c[tok, dim] |= ((page[off] >> sh) & 1).astype(np.int16) << 4
        idx, tok, b = _K_SCALES
        bases = (20480, 22528) if fmt == "q5_1" else (20480,)
        dm = np.zeros((PAGE_TOKENS, N_BLOCKS, len(bases)), dtype=np.uint16)
        for j, base in enumerate(bases):
            dm[tok, b, j] = page[base + 2 * idx].astype(np.uint16) | (page[base + 2 * idx + 1].astype(np.uint16) << 8)
        dm = dm.view(np.float16)
        return c.astype(np.uint8).reshape(PAGE_TOKENS, N_BLOCKS, 32), (dm if fmt == "q5_1" else dm[..., 0])
    if role == "v" and fmt == "q4_1":
        off, tok, lo, hi = _V4_NIBBLES
        c[tok, lo] = page[off] & 0xF
        c[tok, hi] = page[off] >> 4
        idx, tok, b = _V_SCALES
        dm = np.zeros((PAGE_TOKENS, N_BLOCKS, 2), dtype=np.uint16)
        for j, base in enumerate((16384, 18432)):
            dm[tok, b, j] = page[base + 2 * idx].astype(np.uint16) | (page[base + 2 * idx + 1].astype(np.uint16) << 8)
        return c.astype(np.uint8).reshape(PAGE_TOKENS, N_BLOCKS, 32), dm.view(np.float16)
    if role == "k" and fmt == "q4_0":
        off, sh, tok, dim = _K4_NIBBLES
        c[tok, dim] = (page[off] >> sh) & 0xF
        idx, tok, b = _K_SCALES
        scale_base = 16384
    elif role == "k":
        off, tok, dim = _K_CODES
        c[tok, dim] = page[off].astype(np.int16) - 128
        idx, tok, b = _K_SCALES
        scale_base = 32768
    elif fmt == "q4_0":
        off, tok, lo, hi = _V4_NIBBLES
        c[tok, lo] = page[off] & 0xF
        c[tok, hi] = page[off] >> 4
        idx, tok, b = _V_SCALES
        scale_base = 16384
    else:
        off, tok, dim = _V8_CODES
        c[tok, dim] = page[off].astype(np.int16) - 128
        idx, tok, b = _V_SCALES
        scale_base = 32768
    d16 = np.zeros((PAGE_TOKENS, N_BLOCKS), dtype=np.uint16)
    d16[tok, b] = page[scale_base + 2 * idx].astype(np.uint16) | (page[scale_base + 2 * idx + 1].astype(np.uint16) << 8)
    dt = np.int8 if fmt == "q8_0" else np.uint8
    return c.astype(dt).reshape(PAGE_TOKENS, N_BLOCKS, 32), d16.view(np.float16)

"""Pins for the oracle's page byte layout (CPU only).

The layout is this library's own storage spec; the pins are its size (equal to
the pages' block sizes), that encoding is a bijection, and spot values of the
documented offset formulas.
"""
import numpy as np
import pytest

from oracle import layout, quant
from synth import normal_f32, np_rng


def _page(fmt, seed):
    x = normal_f32(np_rng(seed), (128, 256))
    return quant.quantize(x, fmt)


@pytest.mark.parametrize("role,fmt", [("k", "q8_0"), ("k", "q4_0"), ("k", "q5_1"), ("k", "q5_0"), ("v", "q4_0"),
                                      ("v", "q8_0"), ("v", "q4_1")])
def test_round_trip(role, fmt):
    codes, d = _page(fmt, 11)
    page = layout.encode_page(role, fmt, codes, d)
    assert page.size == layout.page_bytes(role, fmt) == 128 * 8 * quant.block_bytes(fmt)
    c2, d2 = layout.decode_page(role, fmt, page)
    assert np.array_equal(c2, codes) and np.array_equal(d2.view(np.uint16), d.view(np.uint16))


def _one_hot(fmt, tok, dim, code):
    """A page of zero bytes but for one code (Q8_0: the code -128 is the zero byte)."""
    codes = np.zeros((128, 8, 32), dtype=np.int8 if fmt == "q8_0" else np.uint8)
    if fmt == "q8_0":
        codes[:] = -128
    codes[tok, dim // 32, dim % 32] = code
    return codes, np.zeros((128, 8), np.float16)


@pytest.mark.parametrize("tok,dim,off", [
    (0, 0, 0), (1, 0, 64), (8, 0, 512), (0, 8, 16), (0, 32, 8), (0, 64, 1024),
    (16, 0, 4096), (5, 200, 3 * 1024 + 5 * 64 + 1 * 16),
])
def test_k_code_offsets(tok, dim, off):
    codes, d = _one_hot("q8_0", tok, dim, 7)
    page = layout.encode_page("k", "q8_0", codes, d)
    assert np.flatnonzero(page).tolist() == [off]
    assert page[off] == 7 + 128


@pytest.mark.parametrize("code,byte", [(-128, 0x00), (-127, 0x01), (-1, 0x7F), (0, 0x80), (1, 0x81), (127, 0xFF)])
def test_q8_codes_are_stored_offset_binary(code, byte):
    for role in ("k", "v"):
        codes, d = _one_hot("q8_0", 3, 77, code)
        page = layout.encode_page(role, "q8_0", codes, d)
        assert page[:32768].tolist().count(byte) == (32768 if code == -128 else 1)
        c2, _ = layout.decode_page(role, "q8_0", page)
        assert c2[3, 2, 13] == code and c2.dtype == np.int8


# K Q4_0: word 4*((((G*2+Q)*2+H)*8+R)*4+T)*4+c) for token 16G+8H+R, block 4Q+c; channel
# 32b+8T+i sits at bit 4*(i//2) + 16*(i%2) of the little-endian word (offsets worked by hand)
@pytest.mark.parametrize("tok,dim,off,shift", [
    (0, 0, 0, 0), (0, 1, 2, 0), (0, 2, 0, 4), (0, 3, 2, 4), (0, 4, 1, 0), (0, 5, 3, 0),
    (0, 6, 1, 4), (0, 7, 3, 4), (0, 8, 16, 0), (0, 32, 4, 0), (0, 128, 1024, 0), (1, 0, 64, 0),
    (8, 0, 512, 0), (16, 0, 2048, 0), (5, 200, 1368, 0),
])
def test_k_q4_nibble_offsets(tok, dim, off, shift):
    codes = np.zeros((128, 8, 32), np.uint8)
    codes[tok, dim // 32, dim % 32] = 9
    page = layout.encode_page("k", "q4_0", codes, np.zeros((128, 8), np.float16))
    assert np.flatnonzero(page).tolist() == [off]
    assert page[off] == 9 << shift


def test_k_q4_scales_follow_the_q8_k_arrangement():
    d = np.zeros((128, 8), np.float16)
    d[9, 3] = 1.0          # same index 27 as the Q8_0 K page, after 16,384 bytes of nibbles
    page = layout.encode_page("k", "q4_0", np.zeros((128, 8, 32), np.uint8), d)
    assert np.flatnonzero(page).tolist() == [16384 + 2 * 27 + 1]


# K Q5_1: bit 4 of the code of token 16G+8H+R, channel 32(4Q+c)+8T+i sits in the word at
# 16384 + 4*((((G*2+Q)*2+H)*8+R)*4+T), bit 16*(i%2) + 4c + i//2 (worked by hand)
@pytest.mark.parametrize("tok,dim,off,bit", [
    (0, 0, 16384, 0), (0, 1, 16386, 0), (0, 2, 16384, 1), (0, 32, 16384, 4), (0, 96, 16385, 4),
    (0, 103, 16387, 7), (0, 8, 16388, 0), (0, 128, 16640, 0), (1, 0, 16400, 0), (8, 0, 16512, 0),
    (16, 0, 16896, 0),
])
def test_k_q5_1_fifth_bit_offsets(tok, dim, off, bit):
    codes = np.zeros((128, 8, 32), np.uint8)
    codes[tok, dim // 32, dim % 32] = 16
    page = layout.encode_page("k", "q5_1", codes, np.zeros((128, 8, 2), np.float16))
    assert np.flatnonzero(page).tolist() == [off]
    assert page[off] == 1 << bit
    codes[tok, dim // 32, dim % 32] = 17      # the low nibble goes where a Q4_0 key nibble goes
    page2 = layout.encode_page("k", "q5_1", codes, np.zeros((128, 8, 2), np.float16))
    nib = layout.encode_page("k", "q4_0", np.where(codes > 0, 1, 0).astype(np.uint8), np.zeros((128, 8), np.float16))
    assert np.array_equal(page2[:16384], nib[:16384]) and np.array_equal(page2[16384:], page[16384:])


def test_k_q5_1_scale_and_minimum_offsets():
    dm = np.zeros((128, 8, 2), np.float16)
    dm[9, 3, 0] = 1.0      # index 27 of the K scale arrangement
    dm[9, 3, 1] = 2.0      # 0x4000
    page = layout.encode_page("k", "q5_1", np.zeros((128, 8, 32), np.uint8), dm)
    assert np.flatnonzero(page).tolist() == [20480 + 2 * 27 + 1, 22528 + 2 * 27 + 1]
    assert page[20480 + 55] == 0x3C and page[22528 + 55] == 0x40


def test_k_q5_0_matches_q5_1_codes_and_scales_without_minima():
    codes = np.zeros((128, 8, 32), np.uint8)
    codes[5, 6, 8], codes[9, 3, 31] = 16, 27
    d = np.zeros((128, 8), np.float16)
    d[9, 3] = 1.0
    dm = np.zeros((128, 8, 2), np.float16)
    dm[..., 0] = d
    p50 = layout.encode_page("k", "q5_0", codes, d)
    p51 = layout.encode_page("k", "q5_1", codes, dm)
    assert p50.size == 22528 and np.array_equal(p50, p51[:22528]) and not p51[22528:].any()


def test_v_q4_1_matches_q4_0_nibbles_and_scales_plus_minima():
    codes = np.zeros((128, 8, 32), np.uint8)
    codes[10, 2, 17] = 6
    dm = np.zeros((128, 8, 2), np.float16)
    dm[10, 2, 0], dm[10, 2, 1] = 1.0, 2.0     # token 10 of block 2 -> scale index 42
    p41 = layout.encode_page("v", "q4_1", codes, dm)
    p40 = layout.encode_page("v", "q4_0", codes, dm[..., 0])
    assert p41.size == 20480 and np.array_equal(p41[:18432], p40)
    assert np.flatnonzero(p41[18432:]).tolist() == [2 * 42 + 1] and p41[18432 + 85] == 0x40


def test_k_scale_offsets():
    codes = np.full((128, 8, 32), -128, np.int8)      # code bytes all zero
    d = np.zeros((128, 8), np.float16)
    d[9, 3] = 1.0          # G=0, R=1, H=1, b=3 -> index ((0*8+1)*2+1)*8+3 = 27
    page = layout.encode_page("k", "q8_0", codes, d)
    nz = np.flatnonzero(page)
    assert nz.tolist() == [32768 + 2 * 27 + 1]     # 1.0 = 0x3C00: only the high byte is set


@pytest.mark.parametrize("tok,dim,off,shift", [
    (0, 0, 0, 0), (0, 8, 0, 4), (0, 16, 1, 0), (0, 24, 1, 4), (1, 0, 2, 0),
    (8, 0, 4, 0), (2, 0, 16, 0), (0, 1, 64, 0), (0, 32, 8, 0), (0, 64, 512, 0), (16, 0, 2048, 0),
])
def test_v_q4_nibble_offsets(tok, dim, off, shift):
    codes = np.zeros((128, 8, 32), np.uint8)
    codes[tok, dim // 32, dim % 32] = 5
    page = layout.encode_page("v", "q4_0", codes, np.zeros((128, 8), np.float16))
    assert np.flatnonzero(page).tolist() == [off]
    assert page[off] == 5 << shift


@pytest.mark.parametrize("tok,dim,off", [
    (0, 0, 0), (1, 0, 1), (0, 8, 2), (8, 0, 4), (0, 16, 8), (2, 0, 16), (0, 1, 64), (0, 32, 512),
    (16, 0, 4096),
])
def test_v_q8_code_offsets(tok, dim, off):
    codes, d = _one_hot("q8_0", tok, dim, 9)
    page = layout.encode_page("v", "q8_0", codes, d)
    assert np.flatnonzero(page).tolist() == [off]
    assert page[off] == 9 + 128


def test_v_scale_offsets():
    d = np.zeros((128, 8), np.float16)
    d[10, 2] = 1.0        # tok 10 = 2T + k%2 + 8*(k//2) with T=1, k=2 -> index ((0*4+1)*8+2)*4+2 = 42
    for fmt, base in (("q4_0", 16384), ("q8_0", 32768)):
        codes = np.zeros((128, 8, 32), np.int8 if fmt == "q8_0" else np.uint8)
        if fmt == "q8_0":
            codes[:] = -128                            # code bytes all zero
        page = layout.encode_page("v", fmt, codes, d)
        assert np.flatnonzero(page).tolist() == [base + 2 * 42 + 1]

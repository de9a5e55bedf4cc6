"""Pins for the oracle's Q8_0 / Q4_0 quantisers (CPU only).

Closed-form error bounds, exact round trips of representable blocks, the
rounding rule at exact halves, the zero block and the scale's fp16 rounding.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import quant
from synth import normal_f32, np_rng


def _x(seed, n_blocks=64, outliers=False):
    x = normal_f32(np_rng(seed), (n_blocks * 32,))
    if outliers:
        x[::37] *= 8.0
    return x


@pytest.mark.parametrize("outliers", [False, True])
def test_q8_0_error_bound(outliers):
    x = _x(1, 256, outliers).reshape(-1, 32)
    qs, d = quant.q8_0_quantize(x)
    xh = quant.q8_0_dequantize(qs, d).reshape(-1, 32)
    d32 = (np.max(np.abs(x), axis=1) / np.float32(127)).astype(np.float32).astype(np.float64)
    d16 = d.astype(np.float64).reshape(-1)
    bound = d32 * (0.5 + 2.0 ** -16) + 127 * np.abs(d32 - d16)
    assert np.all(np.abs(x - xh) <= bound[:, None] + 1e-300)


def test_q8_0_codes_are_nearest_away_from_zero():
    x = _x(2, 128).reshape(-1, 32)
    qs = quant.q8_0_quantize(x)[0].reshape(-1, 32)
    d32 = (np.max(np.abs(x), axis=1) / np.float32(127)).astype(np.float32)
    for i in range(x.shape[0]):
        for j in range(32):
            exact = Fraction(float(x[i, j])) / Fraction(float(d32[i]))
            k = int(np.floor(abs(exact) + Fraction(1, 2))) * (1 if exact >= 0 else -1)
            if abs(abs(exact - int(exact)) - Fraction(1, 2)) > Fraction(1, 10 ** 4):
                assert qs[i, j] == k


def test_q8_0_halves_round_away_from_zero():
    # amax = 15.875 -> d = 0.125 exactly, 1/d = 8 exactly, so x*8 hits exact halves.
    x = np.zeros(32, np.float32)
    x[0] = 15.875
    x[1:5] = [0.0625, 0.3125, -0.3125, -0.0625]   # 0.5, 2.5, -2.5, -0.5
    qs, d = quant.q8_0_quantize(x)
    assert float(d[0]) == 0.125
    assert list(qs[0, :5]) == [127, 1, 3, -3, -1]


def test_q8_0_round_trip_of_representable_block():
    rng = np_rng(3)
    q = rng.integers(-127, 128, size=(16, 32)).astype(np.int8)
    q[:, 5] = 127
    d = np.float16(2.0 ** -4)
    x = (q.astype(np.float32) * np.float32(d))
    qs, dd = quant.q8_0_quantize(x)
    assert np.array_equal(qs.reshape(q.shape), q) and np.all(dd == d)


def test_q8_0_zero_block_and_extremes():
    x = np.zeros(64, np.float32)
    x[40] = -3.0
    qs, d = quant.q8_0_quantize(x)
    assert d[0] == 0 and np.all(qs[0] == 0)
    assert qs[1, 8] == -127


def test_scale_rounds_to_nearest_even_fp16():
    # d = amax/127 = 1 + 2^-11 exactly: halfway between fp16 1.0 and 1.0 + 2^-10.
    x = np.zeros(32, np.float32)
    x[0] = np.float32(127.06201171875)
    _, d = quant.q8_0_quantize(x)
    assert float(d[0]) == 1.0


@pytest.mark.parametrize("outliers", [False, True])
def test_q4_0_error_bound(outliers):
    x = _x(4, 256, outliers).reshape(-1, 32)
    q, d = quant.q4_0_quantize(x)
    assert q.max() <= 15
    xh = quant.q4_0_dequantize(q, d).reshape(-1, 32)
    idx = np.argmax(np.abs(x), axis=1)
    m = x[np.arange(x.shape[0]), idx].astype(np.float64)
    d32 = np.abs(m) / 8.0
    d16 = np.abs(d.astype(np.float64).reshape(-1))
    y = x / (-m[:, None] / 8.0)
    clamped = y >= 7.5 - 1e-6
    tol = np.where(clamped, 1.0, 0.5) + 2.0 ** -18
    bound = d32[:, None] * tol + 8 * np.abs(d32 - d16)[:, None]
    assert np.all(np.abs(x - xh) <= bound)


def test_q4_0_largest_element_maps_to_code_zero():
    x = _x(5, 64).reshape(-1, 32)
    q, d = quant.q4_0_quantize(x)
    q, d = q.reshape(-1, 32), d.reshape(-1)
    idx = np.argmax(np.abs(x), axis=1)
    assert np.all(q[np.arange(x.shape[0]), idx] == 0)
    m = x[np.arange(x.shape[0]), idx]
    assert np.allclose(-8.0 * d.astype(np.float64), m, rtol=2.0 ** -11)


def test_q4_0_round_trip_and_halves():
    rng = np_rng(6)
    d = 0.25
    q = rng.integers(0, 16, size=(8, 32)).astype(np.uint8)
    q[:, 3] = 0                               # value -8d: the largest magnitude
    x = ((q.astype(np.float32) - 8) * np.float32(d))
    qq, dd = quant.q4_0_quantize(x)
    assert np.array_equal(qq.reshape(q.shape), q) and np.all(dd.astype(np.float64) == d)
    # exact halves: y = -0.5 -> code 8, y = +0.5 -> code 9, y = 7.5 -> clamp 15
    x = np.zeros(32, np.float32)
    x[0] = -8 * d
    x[1:4] = [-0.5 * d, 0.5 * d, 7.5 * d]
    qq, _ = quant.q4_0_quantize(x)
    assert list(qq[0, :4]) == [0, 8, 9, 15]


def test_q4_0_zero_block():
    q, d = quant.q4_0_quantize(np.zeros(32, np.float32))
    assert d[0] == 0 and np.all(q == 8)
    assert np.all(quant.q4_0_dequantize(q, d) == 0)


def test_block_bytes_match_bits_per_element():
    assert quant.block_bytes("q8_0") * 8 / 32 == 8.5
    assert quant.block_bytes("q4_0") * 8 / 32 == 4.5
    assert quant.block_bytes("q5_1") * 8 / 32 == 6.0


def test_q5_1_bits_are_a_third_more_than_q4_0():
    # the Vulkan report's pitfalls section: Q5_1 keys give a third more key precision (bits)
    # than Q4_0 keys
    assert Fraction(quant.block_bytes("q5_1"), quant.block_bytes("q4_0")) == Fraction(4, 3)


@pytest.mark.parametrize("outliers", [False, True])
def test_q5_1_error_bound(outliers):
    x = _x(7, 256, outliers).reshape(-1, 32)
    q, dm = quant.q5_1_quantize(x)
    xh = quant.q5_1_dequantize(q, dm).reshape(-1, 32)
    mn = x.min(axis=1).astype(np.float64)
    d32 = ((x.max(axis=1) - x.min(axis=1)).astype(np.float32) / np.float32(31)).astype(np.float32).astype(np.float64)
    d16 = dm[:, 0, 0].astype(np.float64)
    m16 = dm[:, 0, 1].astype(np.float64)
    bound = d32 * (0.5 + 1e-5) + 31 * np.abs(d32 - d16) + np.abs(mn - m16)
    assert np.all(np.abs(x - xh) <= bound[:, None])
    assert np.all(q <= 31)


def test_q5_1_extremes_map_to_codes_0_and_31():
    x = _x(8, 64).reshape(-1, 32)
    q, _ = quant.q5_1_quantize(x)
    q = q.reshape(-1, 32)
    rows = np.arange(x.shape[0])
    assert np.all(q[rows, np.argmin(x, axis=1)] == 0)
    assert np.all(q[rows, np.argmax(x, axis=1)] == 31)


def test_q5_1_round_trip_and_halves():
    rng = np_rng(9)
    d, m = 0.25, -1.0
    q = rng.integers(0, 32, size=(8, 32)).astype(np.uint8)
    q[:, 0], q[:, 1] = 0, 31                   # the block's minimum and maximum
    x = (q.astype(np.float32) * np.float32(d) + np.float32(m)).astype(np.float32)
    qq, dm = quant.q5_1_quantize(x)
    assert np.array_equal(qq.reshape(q.shape), q)
    assert np.all(dm[..., 0].astype(np.float64) == d) and np.all(dm[..., 1].astype(np.float64) == m)
    assert np.array_equal(quant.q5_1_dequantize(qq, dm).reshape(q.shape), x.astype(np.float64))
    # exact halves round up: (x - m) / d = 0.5 -> 1, 30.5 -> 31, 2.25 -> 2
    x = np.zeros(32, np.float32)
    x[0], x[1] = m, m + 31 * d
    x[2:5] = [m + 0.5 * d, m + 30.5 * d, m + 2.25 * d]
    qq, _ = quant.q5_1_quantize(x)
    assert list(qq[0, :5]) == [0, 31, 1, 31, 2]
    assert qq[0, 5] == 4                       # x = 0: (0 - m) / d = 4


def test_q5_1_constant_block():
    q, dm = quant.q5_1_quantize(np.full(32, 1.5, np.float32))
    assert dm[0, 0] == 0 and dm[0, 1] == np.float16(1.5) and np.all(q == 0)
    assert np.all(quant.q5_1_dequantize(q, dm) == 1.5)


def test_q5_0_and_q4_1_bits_per_element():
    assert quant.block_bytes("q5_0") * 8 / 32 == 5.5
    assert quant.block_bytes("q4_1") * 8 / 32 == 5.0


@pytest.mark.parametrize("outliers", [False, True])
def test_q5_0_error_bound(outliers):
    x = _x(10, 256, outliers).reshape(-1, 32)
    q, d = quant.q5_0_quantize(x)
    xh = quant.q5_0_dequantize(q, d).reshape(-1, 32)
    idx = np.argmax(np.abs(x), axis=1)
    m = x[np.arange(x.shape[0]), idx]
    d32 = (m / np.float32(-16)).astype(np.float32).astype(np.float64)
    d16 = d.astype(np.float64).reshape(-1)
    # |x - (q - 16) d32| <= |d32| / 2 (1 at the clamp q = 31) plus rounding slack, then the
    # fp16 scale moves each value by at most 16 |d32 - d16|
    err = np.abs(x - xh)
    bound = np.abs(d32) * (1.0 + 1e-5) + 16 * np.abs(d32 - d16)
    assert np.all(err <= bound[:, None])
    assert np.all(q <= 31)
    # the largest-magnitude element maps to code 0, and m = -16 d up to the fp16 rounding
    assert np.all(q.reshape(-1, 32)[np.arange(x.shape[0]), idx] == 0)
    assert np.allclose(-16.0 * d16, m, rtol=2.0 ** -11)


def test_q5_0_round_trip_halves_and_zero_block():
    rng = np_rng(11)
    d = 0.125
    q = rng.integers(0, 32, size=(8, 32)).astype(np.uint8)
    q[:, 5] = 0                               # value -16 d: the largest magnitude
    x = ((q.astype(np.float32) - 16) * np.float32(d))
    qq, dd = quant.q5_0_quantize(x)
    assert np.array_equal(qq.reshape(q.shape), q) and np.all(dd.astype(np.float64) == d)
    # exact halves: y = -0.5 -> 16, +0.5 -> 17, 15.5 -> clamp 31
    x = np.zeros(32, np.float32)
    x[0] = -16 * d
    x[1:4] = [-0.5 * d, 0.5 * d, 15.5 * d]
    qq, _ = quant.q5_0_quantize(x)
    assert list(qq[0, :4]) == [0, 16, 17, 31]
    q0, d0 = quant.q5_0_quantize(np.zeros(32, np.float32))
    assert d0[0] == 0 and np.all(q0 == 16) and np.all(quant.q5_0_dequantize(q0, d0) == 0)


@pytest.mark.parametrize("outliers", [False, True])
def test_q4_1_error_bound_and_extremes(outliers):
    x = _x(12, 256, outliers).reshape(-1, 32)
    q, dm = quant.q4_1_quantize(x)
    xh = quant.q4_1_dequantize(q, dm).reshape(-1, 32)
    mn = x.min(axis=1).astype(np.float64)
    d32 = ((x.max(axis=1) - x.min(axis=1)).astype(np.float32) / np.float32(15)).astype(np.float32).astype(np.float64)
    d16 = dm[:, 0, 0].astype(np.float64)
    m16 = dm[:, 0, 1].astype(np.float64)
    bound = d32 * (0.5 + 1e-5) + 15 * np.abs(d32 - d16) + np.abs(mn - m16)
    assert np.all(np.abs(x - xh) <= bound[:, None])
    q = q.reshape(-1, 32)
    rows = np.arange(x.shape[0])
    assert np.all(q[rows, np.argmin(x, axis=1)] == 0) and np.all(q[rows, np.argmax(x, axis=1)] == 15)


def test_q4_1_round_trip_halves_and_constant_block():
    rng = np_rng(13)
    d, m = 0.5, -3.0
    q = rng.integers(0, 16, size=(8, 32)).astype(np.uint8)
    q[:, 0], q[:, 1] = 0, 15
    x = (q.astype(np.float32) * np.float32(d) + np.float32(m)).astype(np.float32)
    qq, dm = quant.q4_1_quantize(x)
    assert np.array_equal(qq.reshape(q.shape), q)
    assert np.array_equal(quant.q4_1_dequantize(qq, dm).reshape(q.shape), x.astype(np.float64))
    # exact halves round up: (x - m) / d = 0.5 -> 1, 14.5 -> 15, 6.25 -> 6
    x = np.zeros(32, np.float32)
    x[0], x[1] = m, m + 15 * d
    x[2:5] = [m + 0.5 * d, m + 14.5 * d, m + 6.25 * d]
    qq, _ = quant.q4_1_quantize(x)
    assert list(qq[0, :5]) == [0, 15, 1, 15, 6]
    q0, dm0 = quant.q4_1_quantize(np.full(32, -0.75, np.float32))
    assert dm0[0, 0] == 0 and dm0[0, 1] == np.float16(-0.75) and np.all(q0 == 0)

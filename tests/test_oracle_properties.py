"""Property-based pins of the oracle's quantizers and page layouts (CPU only, hypothesis).

For arbitrary finite fp32 blocks, including ties, repeated values, tiny and huge magnitudes:
codes stay in range, the extreme elements map to the codes the encoder definition fixes, and
the reconstruction error stays within the closed-form bound of each format; and any codes and
scales survive the page byte layout unchanged."""
import numpy as np
import pytest
from hypothesis import assume, given, settings
from hypothesis import strategies as st
from hypothesis.extra.numpy import arrays

from oracle import layout, quant

F32 = np.float32
# magnitudes that keep fp16 scales normal and the block range finite in fp32
finite = st.floats(min_value=-3.0e3, max_value=3.0e3, allow_nan=False, allow_infinity=False, width=32)
blocks = arrays(F32, (4, 32), elements=finite)


def _in_range(x, fmt):
    """The oracle refuses blocks whose fp32 scale has no finite reciprocal."""
    try:
        quant.quantize(x, fmt)
        return True
    except ValueError:
        return False


def _f16_gap(v):
    """|v - fp16(v)| for fp32 values, as float64."""
    v = np.asarray(v, np.float64)
    return np.abs(v - v.astype(np.float16).astype(np.float64))


@settings(max_examples=200, deadline=None)
@given(blocks)
def test_offset_formats_codes_and_bound(x):
    for fmt, half in (("q4_0", 8), ("q5_0", 16)):
        assume(_in_range(x, fmt))
        q, d = quant.quantize(x, fmt)
        assert q.max() <= 2 * half - 1
        xh = quant.dequantize(q, d, fmt).reshape(4, 32)
        idx = np.argmax(np.abs(x), axis=1)
        d32 = (x[np.arange(4), idx] / F32(-half)).astype(F32).astype(np.float64)
        # the element of largest magnitude maps to code 0 whenever the fp32 scale is nonzero
        # (a scale that underflows to zero gives the zero block's codes, q = half)
        nz = d32 != 0
        assert np.all(q.reshape(4, 32)[np.arange(4), idx][nz] == 0)
        assert np.all(q.reshape(4, 32)[~nz] == half)
        bound = np.abs(d32) * (1.0 + 1e-5) + half * _f16_gap(d32)
        assert np.all(np.abs(x - xh) <= bound[:, None] + 1e-30)


@settings(max_examples=200, deadline=None)
@given(blocks)
def test_min_formats_codes_and_bound(x):
    for fmt, top in (("q4_1", 15), ("q5_1", 31)):
        assume(_in_range(x, fmt))
        q, dm = quant.quantize(x, fmt)
        assert q.max() <= top
        qq = q.reshape(4, 32)
        rows = np.arange(4)
        assert np.all(qq[rows, np.argmin(x, axis=1)] == 0)
        d32 = ((x.max(axis=1) - x.min(axis=1)).astype(F32) / F32(top)).astype(F32).astype(np.float64)
        spread = d32 != 0
        assert np.all(qq[rows, np.argmax(x, axis=1)][spread] == top)
        assert np.all(qq[~spread] == 0)
        xh = quant.dequantize(q, dm, fmt).reshape(4, 32)
        mn = x.min(axis=1).astype(np.float64)
        bound = d32 * (0.5 + 1e-5) + top * _f16_gap(d32) + _f16_gap(mn)
        assert np.all(np.abs(x - xh) <= bound[:, None] + 1e-30)


@settings(max_examples=200, deadline=None)
@given(blocks)
def test_q8_0_codes_and_bound(x):
    assume(_in_range(x, "q8_0"))
    q, d = quant.q8_0_quantize(x)
    assert np.abs(q.astype(int)).max() <= 127
    xh = quant.q8_0_dequantize(q, d).reshape(4, 32)
    d32 = (np.abs(x).max(axis=1) / F32(127)).astype(F32).astype(np.float64)
    bound = d32 * (0.5 + 2.0 ** -16) + 127 * _f16_gap(d32)
    assert np.all(np.abs(x - xh) <= bound[:, None] + 1e-30)


PAGES = [("k", "q8_0", 127, False), ("k", "q4_0", 15, False), ("k", "q5_0", 31, False), ("k", "q5_1", 31, True),
         ("v", "q4_0", 15, False), ("v", "q4_1", 15, True), ("v", "q8_0", 127, False)]


@pytest.mark.parametrize("role,fmt,top,paired", PAGES)
@settings(max_examples=20, deadline=None)
@given(seed=st.integers(0, 2 ** 32 - 1))
def test_page_layout_is_a_bijection(role, fmt, top, paired, seed):
    rng = np.random.default_rng(seed)
    if fmt == "q8_0":
        codes = rng.integers(-127, 128, (128, 8, 32)).astype(np.int8)
    else:
        codes = rng.integers(0, top + 1, (128, 8, 32)).astype(np.uint8)
    shape = (128, 8, 2) if paired else (128, 8)
    d = rng.standard_normal(shape).astype(np.float16)
    page = layout.encode_page(role, fmt, codes, d)
    assert page.size == layout.page_bytes(role, fmt) == 128 * 8 * quant.block_bytes(fmt)
    c2, d2 = layout.decode_page(role, fmt, page)
    assert np.array_equal(c2, codes) and np.array_equal(d2.view(np.uint16), d.view(np.uint16))


@pytest.mark.parametrize("fmt", ["q8_0", "q4_0", "q5_0", "q4_1", "q5_1"])
def test_blocks_whose_scale_has_no_reciprocal_are_refused(fmt):
    x = np.zeros(32, F32)
    x[3] = F32(1e-40)                        # a subnormal: amax / 127, m / -8, ... overflow 1/d
    with pytest.raises(ValueError, match="outside the supported input range"):
        quant.quantize(x, fmt)
    quant.quantize(np.zeros(32, F32), fmt)   # the all-zero block stays defined (d = 0)

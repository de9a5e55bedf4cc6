"""Pins for the oracle's block summaries, scores and selection (CPU only).

Summaries against a correctly rounded scalar sum, scores against exact rational
arithmetic, selection against a brute-force rank count, the recent window, and
recall of planted needle blocks.
"""
import math
from fractions import Fraction

import numpy as np

from oracle import quant, select
from synth import needle_blocks, normal_f32, np_rng, plant_needles


def _blocks(seed, nb, outliers=False):
    x = normal_f32(np_rng(seed), (nb, 128, 256))
    if outliers:
        x[..., [3, 100, 201]] *= 8
    qs, d = quant.q8_0_quantize(x)
    return qs, d                        # [nb][128][8][32], [nb][128][8]


def test_summaries_equal_correctly_rounded_mean():
    qs, d = _blocks(21, 3, outliers=True)
    s = select.block_summaries(qs, d)
    k = quant.q8_0_dequantize(qs, d)     # [nb][128][256] float64 (exact products)
    for b in range(3):
        for c in range(0, 256, 7):
            ref = np.float32(math.fsum(k[b, :, c].tolist()) / 128.0)
            assert s[b, c] == ref


def test_q4_0_key_summaries_equal_correctly_rounded_mean():
    x = normal_f32(np_rng(24), (2, 128, 256))
    x[..., [5, 77]] *= 8
    qs, d = quant.q4_0_quantize(x)
    s = select.block_summaries(qs, d, "q4_0")
    k = quant.q4_0_dequantize(qs, d)
    for b in range(2):
        for c in range(0, 256, 5):
            assert s[b, c] == np.float32(math.fsum(k[b, :, c].tolist()) / 128.0)
    # code 3 of a Q4_0 block is the value (3 - 8) * d
    const = select.block_summaries(np.full((1, 128, 8, 32), 3, np.uint8), np.full((1, 128, 8), np.float16(0.5)),
                                   "q4_0")
    assert np.all(const == np.float32(-2.5))


def test_q5_1_key_summaries_equal_correctly_rounded_mean():
    x = normal_f32(np_rng(25), (2, 128, 256))
    x[..., [9, 130]] *= 8
    qs, dm = quant.q5_1_quantize(x)
    s = select.block_summaries(qs, dm, "q5_1")
    k = quant.q5_1_dequantize(qs, dm)
    for b in range(2):
        for c in range(0, 256, 5):
            assert s[b, c] == np.float32(math.fsum(k[b, :, c].tolist()) / 128.0)
    # code 3 with d = 0.5 and m = -4 is the value -2.5
    dm1 = np.zeros((1, 128, 8, 2), np.float16)
    dm1[..., 0], dm1[..., 1] = 0.5, -4.0
    const = select.block_summaries(np.full((1, 128, 8, 32), 3, np.uint8), dm1, "q5_1")
    assert np.all(const == np.float32(-2.5))


def test_q5_0_key_summaries_equal_correctly_rounded_mean():
    x = normal_f32(np_rng(26), (2, 128, 256))
    qs, d = quant.q5_0_quantize(x)
    s = select.block_summaries(qs, d, "q5_0")
    k = quant.q5_0_dequantize(qs, d)
    for b in range(2):
        for c in range(0, 256, 7):
            assert s[b, c] == np.float32(math.fsum(k[b, :, c].tolist()) / 128.0)
    # code 11 of a Q5_0 block is the value (11 - 16) * d
    const = select.block_summaries(np.full((1, 128, 8, 32), 11, np.uint8), np.full((1, 128, 8), np.float16(0.25)),
                                   "q5_0")
    assert np.all(const == np.float32(-1.25))


def test_summary_of_a_constant_block():
    qs = np.full((1, 128, 8, 32), -5, np.int8)
    d = np.full((1, 128, 8), np.float16(0.375))
    assert np.all(select.block_summaries(qs, d) == np.float32(-5 * 0.375))


def test_scores_equal_exact_rational_value():
    rng = np_rng(22)
    S = normal_f32(rng, (5, 256)) * 0.1
    Q = normal_f32(rng, (6, 256))
    sc = select.block_scores(S, Q)
    for b in range(5):
        exact = sum(Fraction(float(Q[j, c])) * Fraction(float(S[b, c])) for j in range(6) for c in range(256))
        assert sc[b] == float(exact)


def test_selection_matches_brute_force_rank():
    rng = np_rng(23)
    scores = rng.standard_normal(300)
    scores[[10, 11]] = scores[12]          # a tie: lower index wins
    n_full, n_total, budget, recent = 290, 293, 40, 30
    sel, gap = select.select_blocks(scores, n_full, n_total, budget, recent)
    n_cand = n_full - recent
    chosen = set()
    for b in range(n_cand):
        better = sum(1 for c in range(n_cand) if scores[c] > scores[b] or (scores[c] == scores[b] and c < b))
        if better < budget:
            chosen.add(b)
    expect = sorted(chosen | set(range(n_cand, n_total)))
    assert sel.tolist() == expect
    assert len(sel) == budget + recent + (n_total - n_full)
    assert np.all(np.diff(sel) > 0)
    assert gap >= 0


def test_selection_edge_cases():
    s = np.arange(10, dtype=np.float64)
    sel, gap = select.select_blocks(s, 10, 10, 20, 3)      # budget exceeds candidates
    assert sel.tolist() == list(range(10)) and gap == math.inf
    sel, _ = select.select_blocks(s, 10, 11, 0, 2)         # budget 0: recent + tail only
    assert sel.tolist() == [8, 9, 10]
    sel, _ = select.select_blocks(s, 10, 10, 2, 50)        # recent larger than history
    assert sel.tolist() == list(range(10))


def test_needle_blocks_are_all_selected():
    rng = np_rng(24)
    nb, g = 300, 6
    x = normal_f32(rng, (nb * 128, 256))
    q = normal_f32(rng, (g, 256))
    needles = needle_blocks(rng, nb - 64, 20)
    plant_needles(x, needles, q.astype(np.float64).sum(0), rng, cosine=0.9)
    qs, d = quant.q8_0_quantize(x.reshape(nb, 128, 256))
    sc = select.block_scores(select.block_summaries(qs, d), q)
    sel, gap = select.select_blocks(sc, nb, nb, 32, 64)
    assert set(needles.tolist()) <= set(sel.tolist())
    assert set(range(nb - 64, nb)) <= set(sel.tolist())
    assert gap > 1e-9 * abs(sc).max()

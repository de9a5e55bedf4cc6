"""Pins for the oracle's attention and log-sum-exp merge (CPU only).

Brute force with scalar loops on tiny inputs, closed-form special cases
(constant V, a single key, identical keys, fully masked rows), invariance under
the page order, causality, and the exactness of the chunked LSE merge.
"""
import math

import numpy as np
import pytest

from oracle import attention
from synth import normal_f32, np_rng


def _brute(q, k, v, kpos, qpos, scale):
    R, T = len(q), len(k)
    o = [[0.0] * len(v[0]) for _ in range(R)]
    lse = []
    for r in range(R):
        s = [sum(float(q[r][c]) * float(k[t][c]) for c in range(len(q[r]))) * scale
             if kpos[t] <= qpos[r] else None for t in range(T)]
        vis = [x for x in s if x is not None]
        if not vis:
            lse.append(-math.inf)
            continue
        m = max(vis)
        w = [math.exp(x - m) if x is not None else 0.0 for x in s]
        tot = math.fsum(w)
        for c in range(len(v[0])):
            o[r][c] = math.fsum(w[t] * float(v[t][c]) for t in range(T)) / tot
        lse.append(m + math.log(tot))
    return np.array(o), np.array(lse)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_tiny(seed):
    rng = np_rng(100 + seed)
    R, T, D = 3, 7, 5
    q, k, v = normal_f32(rng, (R, D)) * 2, normal_f32(rng, (T, D)), normal_f32(rng, (T, D))
    kpos = rng.permutation(T)
    qpos = np.array([2, 6, 4])
    o, lse = attention.attend(q, k, v, kpos, qpos, 0.37)
    ob, lb = _brute(q, k, v, kpos, qpos, 0.37)
    assert np.allclose(o, ob, rtol=1e-13, atol=1e-14)
    assert np.allclose(lse, lb, rtol=1e-13, atol=1e-14)


def test_constant_values_return_the_value():
    rng = np_rng(7)
    q, k = normal_f32(rng, (4, 16)), normal_f32(rng, (50, 16))
    v = np.tile(normal_f32(rng, (1, 16)), (50, 1))
    o, _ = attention.attend(q, k, v, np.arange(50), np.full(4, 49), 1 / 4)
    assert np.allclose(o, v[0][None, :], rtol=1e-14, atol=1e-15)


def test_single_key_returns_its_value_and_score():
    rng = np_rng(8)
    q, k, v = normal_f32(rng, (3, 16)), normal_f32(rng, (1, 16)), normal_f32(rng, (1, 16))
    o, lse = attention.attend(q, k, v, [5], [5, 6, 9], 1 / 4)
    assert np.allclose(o, np.repeat(v.astype(np.float64), 3, 0), rtol=0, atol=0)
    s = q.astype(np.float64) @ k[0].astype(np.float64) / 4
    assert np.allclose(lse, s, rtol=1e-15, atol=1e-15)


def test_identical_keys_return_the_mean_value():
    rng = np_rng(9)
    q = normal_f32(rng, (2, 8))
    k = np.tile(normal_f32(rng, (1, 8)), (9, 1))
    v = normal_f32(rng, (9, 8))
    o, lse = attention.attend(q, k, v, np.arange(9), [8, 8], 0.5)
    assert np.allclose(o, v.astype(np.float64).mean(0)[None, :], rtol=1e-13, atol=1e-15)
    s = q.astype(np.float64) @ k[0].astype(np.float64) * 0.5
    assert np.allclose(lse, s + math.log(9), rtol=1e-14)


def test_order_of_keys_does_not_matter():
    rng = np_rng(10)
    q, k, v = normal_f32(rng, (6, 32)), normal_f32(rng, (64, 32)), normal_f32(rng, (64, 32))
    pos = np.arange(64)
    o1, l1 = attention.attend(q, k, v, pos, np.full(6, 63), 1 / 16)
    p = rng.permutation(64)
    o2, l2 = attention.attend(q, k[p], v[p], pos[p], np.full(6, 63), 1 / 16)
    assert np.allclose(o1, o2, rtol=1e-13, atol=1e-15) and np.allclose(l1, l2, rtol=1e-14)


def test_causality_and_fully_masked_rows():
    rng = np_rng(11)
    q, k, v = normal_f32(rng, (3, 8)), normal_f32(rng, (20, 8)), normal_f32(rng, (20, 8))
    pos = np.arange(100, 120)
    o1, l1 = attention.attend(q, k, v, pos, [105, 119, 99], 1.0)
    k2, v2 = k.copy(), v.copy()
    k2[6:] *= -3
    v2[6:] += 1
    o2, l2 = attention.attend(q, k2, v2, pos, [105, 119, 99], 1.0)
    assert np.array_equal(o1[0], o2[0]) and l1[0] == l2[0]
    assert not np.allclose(o1[1], o2[1])
    assert np.all(o1[2] == 0) and l1[2] == -np.inf


def test_decode_is_verify_with_one_token():
    rng = np_rng(12)
    q, k, v = normal_f32(rng, (24, 16)), normal_f32(rng, (40, 16)), normal_f32(rng, (40, 16))
    pos = np.arange(40)
    qpos = np.repeat(np.arange(36, 40), 6)
    o_all, l_all = attention.attend(q, k, v, pos, qpos, 0.25)
    for t in range(4):
        o, l = attention.attend(q[6 * t:6 * t + 6], k, v, pos, np.full(6, 36 + t), 0.25)
        assert np.array_equal(o, o_all[6 * t:6 * t + 6]) and np.array_equal(l, l_all[6 * t:6 * t + 6])


@pytest.mark.parametrize("chunk", [1, 3, 16, 77, 500])
def test_chunked_merge_equals_single_pass(chunk):
    rng = np_rng(13)
    q, k, v = normal_f32(rng, (5, 32)) * 3, normal_f32(rng, (300, 32)), normal_f32(rng, (300, 32))
    pos = np.arange(300)
    qpos = np.array([299, 150, 10, 0, 299])
    o1, l1 = attention.attend(q, k, v, pos, qpos, 1 / 16)
    o2, l2 = attention.attend_chunked(q, k, v, pos, qpos, 1 / 16, chunk)
    assert np.allclose(o2, o1, rtol=1e-12, atol=1e-14)
    assert np.allclose(l2, l1, rtol=1e-12, atol=1e-14)


def test_merge_of_random_partition_and_empty_parts():
    rng = np_rng(14)
    q, k, v = normal_f32(rng, (4, 16)), normal_f32(rng, (90, 16)), normal_f32(rng, (90, 16))
    pos = np.arange(90)
    qpos = np.full(4, 89)
    o1, l1 = attention.attend(q, k, v, pos, qpos, 0.3)
    cuts = np.sort(rng.choice(np.arange(1, 90), 6, replace=False))
    parts = np.split(rng.permutation(90), cuts)
    os_, ls_ = [], []
    for idx in parts + [np.array([], dtype=np.int64)]:
        o, l = attention.attend(q, k[idx], v[idx], pos[idx], qpos, 0.3)
        os_.append(o)
        ls_.append(l)
    o2, l2 = attention.merge_lse(np.stack(os_), np.stack(ls_))
    assert np.allclose(o2, o1, rtol=1e-12, atol=1e-14) and np.allclose(l2, l1, rtol=1e-13)


def test_merge_of_all_empty_parts():
    o, l = attention.merge_lse(np.zeros((3, 2, 4)), np.full((3, 2), -np.inf))
    assert np.all(o == 0) and np.all(l == -np.inf)

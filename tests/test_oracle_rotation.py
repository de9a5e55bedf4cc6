"""Pins of the Hadamard-rotation oracle: the matrix by its definition, orthonormality, the
invariance of exact attention, and the precision gain on outlier channels that the source
report describes."""
import numpy as np

from oracle import attention as oatt
from oracle.rotation import attend_quantized, hadamard_matrix, rotate, rotation
from synth import np_rng, normal_f32


def test_sylvester_entries():
    assert hadamard_matrix(2).tolist() == [[1.0, 1.0], [1.0, -1.0]]
    h = hadamard_matrix(256)
    i = np.arange(256)
    pop = np.vectorize(lambda a: bin(int(a)).count("1"))(i[:, None] & i[None, :])
    assert np.array_equal(h, np.where(pop % 2 == 0, 1.0, -1.0))


def test_rotation_is_symmetric_orthonormal_involution():
    r = rotation(256)
    assert np.array_equal(r, r.T)
    assert np.allclose(r @ r, np.eye(256), atol=1e-15)
    x = np_rng(1).standard_normal((5, 256))
    assert np.allclose(rotate(rotate(x)), x, atol=1e-13)
    assert np.allclose(np.linalg.norm(rotate(x), axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)


def test_exact_attention_is_unchanged_by_rotation():
    rng = np_rng(2)
    T, R = 300, 6
    k, v, q = rng.standard_normal((T, 256)), rng.standard_normal((T, 256)), rng.standard_normal((R, 256))
    pos, qp = np.arange(T), np.full(R, T - 1)
    o, l = oatt.attend(q, k, v, pos, qp, 1.0 / 16)
    o2, l2 = oatt.attend(rotate(q), rotate(k), rotate(v), pos, qp, 1.0 / 16)
    assert np.allclose(rotate(o2), o, atol=1e-12) and np.allclose(l2, l, atol=1e-12)


def test_rotation_reduces_quantization_error_with_outlier_channels():
    rng = np_rng(3)
    T, R = 2048, 6
    k, v = normal_f32(rng, (T, 256)), normal_f32(rng, (T, 256))
    ch = rng.choice(256, 3, replace=False)
    k[:, ch] *= 8
    v[:, ch] *= 8
    q = normal_f32(rng, (R, 256))
    pos, qp = np.arange(T), np.full(R, T - 1)
    exact, _ = oatt.attend(q, k, v, pos, qp, 1.0 / 16)
    plain, _ = attend_quantized(q, k, v, pos, qp, "q4_0", rotated=False)
    rot, _ = attend_quantized(q, k, v, pos, qp, "q4_0", rotated=True)
    e_plain = np.linalg.norm(plain - exact) / np.linalg.norm(exact)
    e_rot = np.linalg.norm(rot - exact) / np.linalg.norm(exact)
    assert e_rot < 0.8 * e_plain, (e_rot, e_plain)

"""GPU: the Hadamard rotation kernel against the oracle, and the rotated decode pipeline
(rotate K/V before the append, rotate Q, decode, rotate the output back) against the oracle's
rotated pipeline; the precision gain on outlier channels."""
import numpy as np
import pytest
import torch

from helpers_kv import GpuCache, compare
from oracle import attention as oatt
from oracle.rotation import attend_quantized, rotate
from synth import normal_f32, np_rng

pytestmark = pytest.mark.gpu


def test_hadamard_kernel_matches_oracle(kv_gpu):
    rng = np_rng(1800)
    x = normal_f32(rng, (1003, 256))
    x[:, rng.choice(256, 5, replace=False)] *= 30.0
    xd = torch.from_numpy(x).cuda()
    out = torch.empty_like(xd)
    kv_gpu.kvattn_hadamard(xd, out)
    ref = rotate(x)
    got = out.cpu().numpy().astype(np.float64)
    assert np.abs(got - ref).max() <= 4e-6 * np.abs(x).max()
    kv_gpu.kvattn_hadamard(xd)  # in place
    assert np.array_equal(xd.cpu().numpy(), out.cpu().numpy())
    kv_gpu.kvattn_hadamard(xd)  # R R = I
    assert np.abs(xd.cpu().numpy() - x).max() <= 8e-6 * np.abs(x).max()


def _pipeline(kv, k, v, q, v_fmt, rotated):
    H, T = k.shape[1], k.shape[0]
    g = q.shape[1] // H
    cache = GpuCache(H, q.shape[1], (T + 127) // 128, v_fmt)
    kt, vt = torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda()
    qd = torch.from_numpy(q).cuda()
    if rotated:
        kv.kvattn_hadamard(kt)
        kv.kvattn_hadamard(vt)
        kv.kvattn_hadamard(qd)
    cache.append(kt, vt, 0)
    out = torch.empty((1, q.shape[1], 256), device="cuda")
    lse = torch.empty((1, q.shape[1]), device="cuda")
    wsb = kv.kvattn_decode_workspace_size(cache.desc, 1, cache.n_blocks)
    ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda")
    qp = torch.tensor([T - 1], dtype=torch.int32, device="cuda")
    kv.kvattn_decode(cache.desc, qd, 1, qp, cache.page_table, None, None, cache.n_blocks, out, lse, ws, wsb)
    if rotated:
        kv.kvattn_hadamard(out)
    torch.cuda.synchronize()
    assert kv.kvattn_device_error() == 0
    return out.cpu().numpy()[0], lse.cpu().numpy()[0]


@pytest.mark.parametrize("v_fmt", ["q4_0", "q8_0"])
def test_rotated_decode_matches_oracle_and_gains_precision(kv_gpu, v_fmt):
    rng = np_rng(1801)
    H, g, T = 2, 6, 3000
    k, v = normal_f32(rng, (T, H, 256)), normal_f32(rng, (T, H, 256))
    for h in range(H):
        ch = rng.choice(256, 3, replace=False)
        k[:, h, ch] *= 8
        v[:, h, ch] *= 8
    q = normal_f32(rng, (1, H * g, 256))
    o_rot, l_rot = _pipeline(kv_gpu, k, v, q, v_fmt, True)
    o_plain, _ = _pipeline(kv_gpu, k, v, q, v_fmt, False)
    pos = np.arange(T)
    e_rot = e_plain = 0.0
    for h in range(H):
        rows = q[0, h * g:(h + 1) * g]
        o_ref, l_ref = attend_quantized(rows, k[:, h], v[:, h], pos, np.full(g, T - 1), v_fmt, rotated=True)
        compare(o_rot[None, h * g:(h + 1) * g], l_rot[None, h * g:(h + 1) * g], o_ref[None], l_ref[None])
        exact, _ = oatt.attend(rows, k[:, h], v[:, h], pos, np.full(g, T - 1), 1.0 / 16)
        e_rot += float(np.linalg.norm(o_rot[h * g:(h + 1) * g] - exact) ** 2)
        e_plain += float(np.linalg.norm(o_plain[h * g:(h + 1) * g] - exact) ** 2)
    assert e_rot < 0.8 ** 2 * e_plain, (e_rot, e_plain)

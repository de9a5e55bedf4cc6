"""GPU: the Q8_0 / Q4_0 encoders write exactly the oracle's bytes (bit-exact)."""
import numpy as np
import pytest
import torch

from helpers_kv import GpuCache, OracleCache
from synth import normal_f32, np_rng, page_permutation

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("k_fmt,v_fmt", [("q8_0", "q4_0"), ("q8_0", "q8_0"), ("q4_0", "q4_0"), ("q4_0", "q8_0"),
                                         ("q5_1", "q4_0"), ("q5_1", "q8_0"), ("q5_0", "q4_1")])
def test_append_bytes_bit_exact(kv_gpu, k_fmt, v_fmt):
    rng = np_rng(501)
    H, T, n_blocks = 4, 3 * 128 + 50, 5
    k = normal_f32(rng, (T, H, 256))
    v = normal_f32(rng, (T, H, 256))
    k[:, :, [3, 100, 201]] *= 8            # outlier channels
    v[:, :, [7, 64]] *= 8
    k[5, 0] = 0.0                            # zero rows -> d = 0
    v[5, 1] = 0.0
    k[9, 2, :32] = 0.0                       # exact halves under d = 0.125 (1/d = 8)
    k[9, 2, 0] = 15.875
    k[9, 2, 1:5] = [0.0625, 0.3125, -0.3125, -0.0625]
    v[9, 3, :32] = 0.0                       # Q4_0 halves: m = -2 -> d = 0.25
    v[9, 3, 0] = -2.0
    v[9, 3, 1:4] = [-0.125, 0.125, 1.875]
    v[11, 0, :32] = 3.0                      # ties of the largest magnitude: first index wins
    v[11, 0, 4] = -3.0
    k[13, 1, 32:64] = 0.0                    # Q5_1 halves: m = -1, d = 0.25, (x - m) / d = k + 0.5
    k[13, 1, 32:37] = [-1.0, 6.75, -0.875, 6.625, -0.4375]
    k[15, 3, 64:96] = 0.0                    # Q5_0 halves: m = -4, d = 0.25, x / d + 16.5 = q + 1
    k[15, 3, 64:68] = [-4.0, 0.125, -0.375, 3.625]
    v[15, 2, 96:128] = 0.5                   # Q4_1: a constant block gives d = 0, q = 0, m = 0.5
    v[17, 2, 0:32] = 0.0                     # Q4_1 halves: m = -1, d = 0.25, (x - m) / d + 0.5 = k + 1
    v[17, 2, 0:6] = [-1.0, 2.75, -0.875, -0.125, 0.875, 2.625]
    n_phys = H * n_blocks + 3
    cache = GpuCache(H, 24, n_blocks, v_fmt, n_phys=n_phys, perm=page_permutation(rng, n_phys), k_fmt=k_fmt)
    for a, b in ((0, 100), (100, 101), (101, 300), (300, T)):
        cache.append(k[a:b], v[a:b], a)
    torch.cuda.synchronize()
    oc = OracleCache(k, v, v_fmt, k_fmt)
    kp = cache.k_pool.cpu().numpy()
    vp = cache.v_pool.cpu().numpy()
    used = set()
    for h in range(H):
        for blk in range((T + 127) // 128):
            pg = int(cache.page_table_np[h, blk])
            used.add(pg)
            assert np.array_equal(kp[pg], oc.page_bytes(h, blk, "k")), (h, blk, "k")
            assert np.array_equal(vp[pg], oc.page_bytes(h, blk, "v")), (h, blk, "v")
    for pg in set(range(n_phys)) - used:
        assert not kp[pg].any() and not vp[pg].any()


def test_append_rejects_blocks_past_the_table(kv_gpu):
    cache = GpuCache(1, 6, 2)
    x = torch.zeros((1, 1, 256), device="cuda")
    with pytest.raises(kv_gpu.KVAttnError) as e:
        kv_gpu.kvattn_quantize_append(cache.desc, x, x, 1, 256, cache.page_table, 2)
    assert e.value.status == kv_gpu.ERR_INVALID_ARG


def test_append_bad_page_id_is_reported(kv_gpu):
    cache = GpuCache(1, 6, 2)
    cache.page_table[0, 1] = 999
    x = torch.ones((1, 1, 256), device="cuda")
    kv_gpu.kvattn_quantize_append(cache.desc, x, x, 1, 130, cache.page_table, 2)
    assert kv_gpu.kvattn_device_error() == kv_gpu.ERR_BAD_PAGE
    assert not cache.k_pool.any()

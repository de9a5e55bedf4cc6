"""GPU: kvattn_decode_noalloc, the decode entry point for callers that cannot allocate device
memory (its scratch is a fixed array inside the library), gives the same results as
kvattn_decode with a caller workspace, on two calls in a row.  Collected last on purpose."""
import numpy as np
import pytest
import torch

from helpers_kv import GpuCache
from synth import normal_f32, np_rng, page_permutation

pytestmark = pytest.mark.gpu


def _cache(seed, H, T):
    rng = np_rng(seed)
    k = normal_f32(rng, (T, H, 256))
    v = normal_f32(rng, (T, H, 256))
    nb = (T + 127) // 128
    cache = GpuCache(H, 6 * H, nb, "q4_0", n_phys=H * nb, perm=page_permutation(rng, H * nb))
    cache.append(k, v, 0)
    return rng, cache, nb


@pytest.mark.parametrize("n_q", [1, 4])
def test_noalloc_decode_matches_decode(kv_gpu, n_q):
    H, T = 4, 37 * 128 + 77
    rng, cache, nb = _cache(9100 + n_q, H, T)
    q_pos = torch.arange(T - n_q, T, dtype=torch.int32, device="cuda")
    wsb = kv_gpu.kvattn_decode_workspace_size(cache.desc, n_q, nb)
    ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda")
    for call in range(2):
        q = torch.from_numpy(normal_f32(rng, (n_q, 6 * H, 256))).cuda()
        ref_o = torch.empty((n_q, 6 * H, 256), device="cuda")
        ref_l = torch.empty((n_q, 6 * H), device="cuda")
        kv_gpu.kvattn_decode(cache.desc, q, n_q, q_pos, cache.page_table, None, None, nb, ref_o, ref_l, ws, wsb)
        out = torch.full((n_q, 6 * H, 256), float("nan"), device="cuda")
        lse = torch.full((n_q, 6 * H), float("nan"), device="cuda")
        kv_gpu.kvattn_decode_noalloc(cache.desc, q, n_q, q_pos, cache.page_table, None, None, nb, out, lse)
        torch.cuda.synchronize()
        # the same kernels with the same split plan: bit-identical results
        assert np.array_equal(out.cpu().numpy(), ref_o.cpu().numpy()), call
        assert np.array_equal(lse.cpu().numpy(), ref_l.cpu().numpy()), call


def test_noalloc_refuses_unsupported_shape_untouched(kv_gpu):
    """GQA 6 with 5 query tokens (30 rows per KV head) is refused as an unsupported shape, as
    kvattn_decode refuses it, and the outputs are left untouched."""
    H, T, n_q = 1, 300, 5
    rng, cache, nb = _cache(9200, H, T)
    q = torch.from_numpy(normal_f32(rng, (n_q, 6 * H, 256))).cuda()
    q_pos = torch.arange(T - n_q, T, dtype=torch.int32, device="cuda")
    out = torch.full((n_q, 6 * H, 256), 7.0, device="cuda")
    lse = torch.full((n_q, 6 * H), 7.0, device="cuda")
    with pytest.raises(kv_gpu.KVAttnError) as e:
        kv_gpu.kvattn_decode_noalloc(cache.desc, q, n_q, q_pos, cache.page_table, None, None, nb, out, lse)
    assert e.value.status == kv_gpu.ERR_UNSUPPORTED_SHAPE
    torch.cuda.synchronize()
    assert bool((out == 7.0).all()) and bool((lse == 7.0).all())

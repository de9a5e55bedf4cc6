"""GPU: split-KV decode / MTP verify against the oracle (max abs 2e-3, relative gate)."""
import numpy as np
import pytest
import torch

from helpers_kv import GpuCache, OracleCache, compare
from synth import normal_f32, np_rng, page_permutation

pytestmark = pytest.mark.gpu


def _layer(seed, H, T, v_fmt, n_blocks=None, spare=0, outliers=True, k_fmt="q8_0"):
    rng = np_rng(seed)
    k = normal_f32(rng, (T, H, 256))
    v = normal_f32(rng, (T, H, 256))
    if outliers:
        for h in range(H):
            ch = rng.choice(256, 3, replace=False)
            k[:, h, ch] *= 8
            v[:, h, ch] *= 8
    n_blocks = n_blocks or (T + 127) // 128
    n_phys = H * n_blocks + spare
    cache = GpuCache(H, 6 * H, n_blocks, v_fmt, n_phys=n_phys, perm=page_permutation(rng, n_phys), k_fmt=k_fmt)
    return rng, k, v, cache


def _run_decode(kv, cache, H_q, q, q_pos, page_list, page_logical=None, n_pages=None, max_pages=None):
    cache.desc.n_q_heads = H_q
    n_q = q.shape[0]
    max_pages = page_list.shape[1] if max_pages is None else max_pages
    qd = torch.from_numpy(np.ascontiguousarray(q)).cuda()
    qp = torch.tensor(q_pos, dtype=torch.int32, device="cuda")
    out = torch.full((n_q, H_q, 256), float("nan"), device="cuda")
    lse = torch.full((n_q, H_q), float("nan"), device="cuda")
    wsb = kv.kvattn_decode_workspace_size(cache.desc, n_q, max_pages)
    ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda")
    pl = torch.as_tensor(page_list, dtype=torch.int32).cuda() if page_list is not None else None
    lg = torch.as_tensor(page_logical, dtype=torch.int32).cuda() if page_logical is not None else None
    npg = torch.as_tensor(n_pages, dtype=torch.int32).cuda() if n_pages is not None else None
    kv.kvattn_decode(cache.desc, qd, n_q, qp, pl, lg, npg, max_pages, out, lse, ws, wsb)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy(), (qd, qp, pl, lg, npg, out, lse, ws, wsb)


FORMAT_PAIRS = [("q8_0", "q4_0"), ("q8_0", "q8_0"), ("q4_0", "q4_0"), ("q4_0", "q8_0"), ("q5_1", "q4_0"),
                ("q5_1", "q8_0"), ("q5_0", "q4_1")]


@pytest.mark.parametrize("k_fmt,v_fmt", FORMAT_PAIRS)
@pytest.mark.parametrize("n_q", [1, 2, 3, 4])
def test_decode_matches_oracle(kv_gpu, k_fmt, v_fmt, n_q):
    H, H_q, T = 4, 24, 37 * 128 + 77          # ragged tail page
    rng, k, v, cache = _layer(600 + n_q, H, T, v_fmt, spare=5, k_fmt=k_fmt)
    cache.append(k, v, 0)
    q = normal_f32(rng, (n_q, H_q, 256))
    q_pos = [T - n_q + i for i in range(n_q)]
    out, lse, keep = _run_decode(kv_gpu, cache, H_q, q, q_pos, cache.page_table_np)
    oc = OracleCache(k, v, v_fmt, k_fmt)
    for h in range(H):
        o_ref, l_ref = oc.attend(q, q_pos, h, 6)
        compare(out[:, 6 * h:6 * h + 6], lse[:, 6 * h:6 * h + 6], o_ref, l_ref)
    # a second launch reusing the workspace gives the same bits
    qd, qp, pl, lg, npg, o2, l2, ws, wsb = keep
    kv_gpu.kvattn_decode(cache.desc, qd, n_q, qp, pl, lg, npg, pl.shape[1], o2, l2, ws, wsb)
    torch.cuda.synchronize()
    assert np.array_equal(o2.cpu().numpy(), out) and np.array_equal(l2.cpu().numpy(), lse)


@pytest.mark.parametrize("k_fmt,v_fmt", [("q8_0", "q4_0"), ("q5_1", "q8_0"), ("q5_0", "q4_1")])
@pytest.mark.parametrize("n_q,T,budget", [(1, 3 * 128 + 40, 148), (1, 37 * 128 + 77, 24), (1, 37 * 128 + 77, 9),
                                          (4, 5 * 128 + 3, 148), (4, 37 * 128 + 77, 20)])
def test_decode_tile_splits_and_sm_budget(kv_gpu, k_fmt, v_fmt, n_q, T, budget):
    """Splits are ranges of 16-token tiles: with few pages over many splits most CTAs take part
    of a page (copied region by region) or nothing at all; a descriptor's SM budget gives fewer
    splits.  Every partition must agree with the oracle."""
    H, H_q = 4, 24
    rng, k, v, cache = _layer(680 + T % 97 + budget, H, T, v_fmt, spare=3, k_fmt=k_fmt)
    cache.append(k, v, 0)
    cache.desc.sm_budget = budget
    q = normal_f32(rng, (n_q, H_q, 256))
    q_pos = [T - n_q + i for i in range(n_q)]
    out, lse, _ = _run_decode(kv_gpu, cache, H_q, q, q_pos, cache.page_table_np)
    assert kv_gpu.kvattn_device_error() == 0
    oc = OracleCache(k, v, v_fmt, k_fmt)
    for h in range(H):
        o_ref, l_ref = oc.attend(q, q_pos, h, 6)
        compare(out[:, 6 * h:6 * h + 6], lse[:, 6 * h:6 * h + 6], o_ref, l_ref)


@pytest.mark.parametrize("n_q", [1, 4])
def test_split_and_merge_calls_equal_decode(kv_gpu, n_q):
    """kvattn_decode_splits then kvattn_decode_merge_splits: bit-identical to kvattn_decode."""
    H, H_q, T = 4, 24, 20 * 128 + 9
    rng, k, v, cache = _layer(650 + n_q, H, T, "q4_0")
    cache.append(k, v, 0)
    q = normal_f32(rng, (n_q, H_q, 256))
    q_pos = [T - n_q + i for i in range(n_q)]
    out, lse, keep = _run_decode(kv_gpu, cache, H_q, q, q_pos, cache.page_table_np)
    qd, qp, pl, lg, npg, o2, l2, ws, wsb = keep
    o2.fill_(float("nan"))
    l2.fill_(float("nan"))
    kv_gpu.kvattn_decode_splits(cache.desc, qd, n_q, qp, pl, lg, npg, pl.shape[1], o2, l2, ws, wsb)
    kv_gpu.kvattn_decode_merge_splits(cache.desc, n_q, pl.shape[1], o2, l2, ws, wsb)
    torch.cuda.synchronize()
    assert np.array_equal(o2.cpu().numpy(), out) and np.array_equal(l2.cpu().numpy(), lse)


@pytest.mark.parametrize("k_fmt,v_fmt", FORMAT_PAIRS)
@pytest.mark.parametrize("n_new,subset", [(1, False), (4, False), (4, True)])
def test_append_decode_equals_append_then_decode(kv_gpu, k_fmt, v_fmt, n_new, subset):
    """kvattn_append_decode against kvattn_quantize_append + kvattn_decode on a copy of the same
    cache: bit-identical outputs and pages.  Four new tokens straddle a page boundary; with
    `subset` the decode lists only some of the older pages, so the new tokens' pages are written
    but not attended."""
    H, H_q, T0 = 4, 24, 20 * 128 + 126
    rng, k, v, cache = _layer(660 + n_new, H, T0 + n_new, v_fmt, spare=3, k_fmt=k_fmt)
    cache.append(k[:T0], v[:T0], 0)
    kp2, vp2 = cache.k_pool.clone(), cache.v_pool.clone()
    desc2 = kv_gpu.make_desc(H, H_q, kp2, vp2, cache.n_phys, v_fmt=v_fmt, k_fmt=k_fmt)
    nb = cache.n_blocks
    k_new = torch.from_numpy(np.ascontiguousarray(k[T0:])).cuda()
    v_new = torch.from_numpy(np.ascontiguousarray(v[T0:])).cuda()
    q = torch.from_numpy(normal_f32(rng, (n_new, H_q, 256))).cuda()
    qp = torch.arange(T0, T0 + n_new, dtype=torch.int32, device="cuda")
    if subset:
        blocks = np.sort(rng.choice(nb - 2, 9, replace=False))
        pl = torch.from_numpy(np.ascontiguousarray(cache.page_table_np[:, blocks])).cuda()
        lg = torch.from_numpy(np.tile(blocks.astype(np.int32), (H, 1))).cuda()
    else:
        pl, lg = cache.page_table, None
    mp = pl.shape[1]
    wsb = kv_gpu.kvattn_decode_workspace_size(cache.desc, n_new, mp)
    outs = []
    for fused, desc in ((False, cache.desc), (True, desc2)):
        ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda")
        out = torch.full((n_new, H_q, 256), float("nan"), device="cuda")
        lse = torch.full((n_new, H_q), float("nan"), device="cuda")
        if fused:
            kv_gpu.kvattn_append_decode(desc, k_new, v_new, n_new, T0, cache.page_table, nb, q, n_new, qp, pl, lg,
                                        None, mp, out, lse, ws, wsb)
        else:
            kv_gpu.kvattn_quantize_append(desc, k_new, v_new, n_new, T0, cache.page_table, nb)
            kv_gpu.kvattn_decode(desc, q, n_new, qp, pl, lg, None, mp, out, lse, ws, wsb)
        torch.cuda.synchronize()
        outs.append((out.cpu().numpy(), lse.cpu().numpy()))
    assert kv_gpu.kvattn_device_error() == 0
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    assert torch.equal(cache.k_pool, kp2) and torch.equal(cache.v_pool, vp2)
    if not subset:
        oc = OracleCache(k, v, v_fmt, k_fmt)
        qn = q.cpu().numpy()
        for h in range(H):
            o_ref, l_ref = oc.attend(qn, list(range(T0, T0 + n_new)), h, 6)
            compare(outs[1][0][:, 6 * h:6 * h + 6], outs[1][1][:, 6 * h:6 * h + 6], o_ref, l_ref)


def test_append_decode_rejects_bad_arguments(kv_gpu):
    rng, k, v, cache = _layer(670, 1, 300, "q4_0", n_blocks=3)
    x = torch.zeros((1, 1, 256), device="cuda")
    q = torch.zeros((1, 6, 256), device="cuda")
    qp = torch.tensor([300], dtype=torch.int32, device="cuda")
    out = torch.empty((1, 6, 256), device="cuda")
    lse = torch.empty((1, 6), device="cuda")
    wsb = kv_gpu.kvattn_decode_workspace_size(cache.desc, 1, 3)
    ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda")
    for n_new, pos0 in ((0, 300), (9, 300), (1, 3 * 128)):   # none, too many, past the table
        with pytest.raises(kv_gpu.KVAttnError) as e:
            kv_gpu.kvattn_append_decode(cache.desc, x, x, n_new, pos0, cache.page_table, 3, q, 1, qp,
                                        cache.page_table, None, None, 3, out, lse, ws, wsb)
        assert e.value.status == kv_gpu.ERR_INVALID_ARG


def test_tiny_workload(kv_gpu):
    # 1 layer, 1 KV head, 6 query heads, 4,096 tokens in 32 shuffled pages, 1 query token
    rng, k, v, cache = _layer(1001, 1, 4096, "q4_0", outliers=False)
    cache.append(k, v, 0)
    q = normal_f32(rng, (1, 6, 256))
    out, lse, _ = _run_decode(kv_gpu, cache, 6, q, [4095], cache.page_table_np)
    o_ref, l_ref = OracleCache(k, v, "q4_0").attend(q, [4095], 0, 6)
    compare(out, lse, o_ref, l_ref)


def test_page_subsets_in_any_order(kv_gpu):
    H, H_q, T = 4, 24, 20 * 128
    rng, k, v, cache = _layer(700, H, T, "q4_0")
    cache.append(k, v, 0)
    q = normal_f32(rng, (1, H_q, 256))
    max_pages = 12
    counts = [12, 7, 1, 0]
    plist = np.zeros((H, max_pages), np.int32)
    plog = np.zeros((H, max_pages), np.int32)
    chosen = []
    for h in range(H):
        blocks = rng.choice(20, counts[h], replace=False)
        chosen.append(blocks)
        plog[h, :counts[h]] = blocks
        plist[h, :counts[h]] = cache.page_table_np[h, blocks]
        plist[h, counts[h]:] = 10 ** 6            # never read: beyond n_pages[h]
    out, lse, _ = _run_decode(kv_gpu, cache, H_q, q, [T - 1], plist, plog, counts, max_pages)
    oc = OracleCache(k, v, "q4_0")
    for h in range(H):
        keys = (chosen[h][:, None] * 128 + np.arange(128)[None, :]).ravel()
        o_ref, l_ref = oc.attend(q, [T - 1], h, 6, key_idx=keys)
        compare(out[:, 6 * h:6 * h + 6], lse[:, 6 * h:6 * h + 6], o_ref, l_ref)
    assert np.all(out[:, 18:] == 0) and np.all(np.isneginf(lse[:, 18:]))


def test_causal_and_fully_masked_rows(kv_gpu):
    H, H_q, T = 2, 12, 9 * 128
    rng, k, v, cache = _layer(710, H, T, "q4_0")
    cache.append(k, v, 0)
    q = normal_f32(rng, (4, H_q, 256))
    q_pos = [3 * 128 + 5, 0, -1, T - 1]        # early, first key only, nothing visible, everything
    out, lse, _ = _run_decode(kv_gpu, cache, H_q, q, q_pos, cache.page_table_np)
    oc = OracleCache(k, v, "q4_0")
    for h in range(H):
        o_ref, l_ref = oc.attend(q, q_pos, h, 6)
        compare(out[:, 6 * h:6 * h + 6], lse[:, 6 * h:6 * h + 6], o_ref, l_ref)
    assert np.all(out[2] == 0) and np.all(np.isneginf(lse[2]))


@pytest.mark.parametrize("k_fmt,v_fmt", FORMAT_PAIRS)
@pytest.mark.parametrize("n_q", [1, 4])
def test_single_short_page_and_empty_list(kv_gpu, k_fmt, v_fmt, n_q):
    """Five keys with x8 outlier channels: outputs of magnitude up to ~25 that average few
    values, the case where f16 rounding of any operand would show."""
    rng, k, v, cache = _layer(720, 1, 5, v_fmt, n_blocks=1, k_fmt=k_fmt)
    cache.append(k, v, 0)
    q = normal_f32(rng, (n_q, 6, 256))
    q_pos = [5 - n_q + i for i in range(n_q)]
    out, lse, _ = _run_decode(kv_gpu, cache, 6, q, q_pos, cache.page_table_np)
    o_ref, l_ref = OracleCache(k, v, v_fmt, k_fmt).attend(q, q_pos, 0, 6)
    compare(out, lse, o_ref, l_ref)
    out, lse, _ = _run_decode(kv_gpu, cache, 6, q, q_pos, np.zeros((1, 1), np.int32), n_pages=[0], max_pages=1)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_bad_page_id_is_reported(kv_gpu):
    rng, k, v, cache = _layer(730, 1, 256, "q4_0")
    cache.append(k, v, 0)
    q = normal_f32(rng, (1, 6, 256))
    plist = cache.page_table_np.copy()
    plist[0, 1] = 12345
    _run_decode(kv_gpu, cache, 6, q, [255], plist)
    assert kv_gpu.kvattn_device_error() == kv_gpu.ERR_BAD_PAGE


def test_rejects_unsupported_shapes(kv_gpu):
    rng, k, v, cache = _layer(740, 1, 128, "q4_0")
    with pytest.raises(kv_gpu.KVAttnError) as e:
        _run_decode(kv_gpu, cache, 6, normal_f32(rng, (5, 6, 256)), [127] * 5, cache.page_table_np)
    assert e.value.status == kv_gpu.ERR_UNSUPPORTED_SHAPE

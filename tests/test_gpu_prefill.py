"""GPU: tcgen05 chunked prefill against the oracle (causal, split across KV, LSE-merged)."""
import numpy as np
import pytest
import torch

from helpers_kv import GpuCache, OracleCache, compare
from synth import bf16_bits, bf16_round, normal_f32, np_rng, page_permutation

pytestmark = pytest.mark.gpu


def _prefill(kv, cache, H_q, q, q_pos, page_list, split, page_logical=None, n_pages=None, max_pages=None,
             f16=False):
    cache.desc.n_q_heads = H_q
    n_q = q.shape[0]
    max_pages = page_list.shape[1] if max_pages is None else max_pages
    qb = torch.from_numpy(bf16_bits(q).view(np.int16)).cuda()
    qp = torch.as_tensor(np.asarray(q_pos, np.int32)).cuda()
    out = torch.full((n_q, H_q, 256), float("nan"), device="cuda")
    lse = torch.full((n_q, H_q), float("nan"), device="cuda")
    wsb = kv.kvattn_prefill_workspace_size(cache.desc, n_q, max_pages, split)
    ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda")
    pl = torch.as_tensor(page_list, dtype=torch.int32).cuda()
    lg = torch.as_tensor(page_logical, dtype=torch.int32).cuda() if page_logical is not None else None
    npg = torch.as_tensor(n_pages, dtype=torch.int32).cuda() if n_pages is not None else None
    call = kv.kvattn_prefill_chunk_f16 if f16 else kv.kvattn_prefill_chunk
    call(cache.desc, qb, n_q, qp, pl, lg, npg, max_pages, split, out, lse, ws, wsb)
    torch.cuda.synchronize()
    assert kv.kvattn_device_error() == 0
    return out.cpu().numpy(), lse.cpu().numpy()


def _case(seed, H, n_prior, n_q, outliers=True, k_fmt="q8_0", v_fmt="q4_0"):
    rng = np_rng(seed)
    T = n_prior + n_q
    k = normal_f32(rng, (T, H, 256))
    v = normal_f32(rng, (T, H, 256))
    if outliers:
        for h in range(H):
            ch = rng.choice(256, 3, replace=False)
            k[:, h, ch] *= 8
            v[:, h, ch] *= 8
    n_blocks = (T + 127) // 128
    n_phys = H * n_blocks + 3
    cache = GpuCache(H, 6 * H, n_blocks, v_fmt, n_phys=n_phys, perm=page_permutation(rng, n_phys), k_fmt=k_fmt)
    cache.append(k, v, 0)
    q = bf16_round(normal_f32(rng, (n_q, 6 * H, 256)))
    return rng, k, v, q, cache, T


PAIRS = [("q8_0", "q4_0"), ("q4_0", "q4_0"), ("q5_1", "q4_0"), ("q5_0", "q4_1"), ("q8_0", "q8_0"), ("q4_0", "q8_0"),
         ("q5_1", "q8_0")]


@pytest.mark.parametrize("k_fmt,v_fmt", PAIRS)
@pytest.mark.parametrize("n_prior,n_q,split", [(700, 40, 256), (1024, 64, 128), (300, 22, 512), (5000, 130, 1024),
                                               (0, 30, 128), (127, 1, 256)])
def test_prefill_matches_oracle(kv_gpu, n_prior, n_q, split, k_fmt, v_fmt):
    """x8 outlier channels and short contexts: outputs of magnitude up to ~25 that average few
    values, where the rounding of any f16 operand would show."""
    H = 2
    rng, k, v, q, cache, T = _case(1200 + n_prior + n_q, H, n_prior, n_q, k_fmt=k_fmt, v_fmt=v_fmt)
    q_pos = np.arange(n_prior, T)
    out, lse = _prefill(kv_gpu, cache, 6 * H, q, q_pos, cache.page_table_np, split)
    oc = OracleCache(k, v, v_fmt, k_fmt)
    for h in range(H):
        o_ref, l_ref = oc.attend(q, q_pos, h, 6)
        compare(out[:, 6 * h:6 * h + 6], lse[:, 6 * h:6 * h + 6], o_ref, l_ref)


@pytest.mark.parametrize("k_fmt,v_fmt", PAIRS)
@pytest.mark.parametrize("n_prior,n_q,split", [(700, 40, 256), (5000, 130, 1024), (0, 30, 128), (4096, 512, 4096)])
def test_prefill_f16_matches_oracle(kv_gpu, n_prior, n_q, split, k_fmt, v_fmt):
    """The one-rounding operand mode on the prefill workload's distribution (K, V and Q drawn
    N(0, 1), no outlier channels): within the same absolute bound as the exact mode."""
    H = 2
    rng, k, v, q, cache, T = _case(1700 + n_prior + n_q, H, n_prior, n_q, outliers=False, k_fmt=k_fmt, v_fmt=v_fmt)
    q_pos = np.arange(n_prior, T)
    out, lse = _prefill(kv_gpu, cache, 6 * H, q, q_pos, cache.page_table_np, split, f16=True)
    oc = OracleCache(k, v, v_fmt, k_fmt)
    for h in range(H):
        o_ref, l_ref = oc.attend(q, q_pos, h, 6)
        compare(out[:, 6 * h:6 * h + 6], lse[:, 6 * h:6 * h + 6], o_ref, l_ref)


def test_prefill_page_subsets(kv_gpu):
    H, n_prior, n_q = 2, 2048, 48
    rng, k, v, q, cache, T = _case(1300, H, n_prior, n_q)
    nb = cache.n_blocks
    keep = [np.sort(rng.choice(nb - 1, 9, replace=False)).tolist() + [nb - 1], list(range(nb))]
    max_pages = max(len(x) for x in keep)
    plist = np.full((H, max_pages), 10 ** 7, np.int32)
    plog = np.zeros((H, max_pages), np.int32)
    for h in range(H):
        order = rng.permutation(len(keep[h]))
        blocks = np.asarray(keep[h])[order]
        plist[h, :len(blocks)] = cache.page_table_np[h, blocks]
        plog[h, :len(blocks)] = blocks
    q_pos = np.arange(n_prior, T)
    out, lse = _prefill(kv_gpu, cache, 6 * H, q, q_pos, plist, 256, plog, [len(x) for x in keep], max_pages)
    oc = OracleCache(k, v, "q4_0")
    for h in range(H):
        keys = (np.asarray(keep[h])[:, None] * 128 + np.arange(128)[None, :]).ravel()
        keys = keys[keys < T]
        o_ref, l_ref = oc.attend(q, q_pos, h, 6, key_idx=keys)
        compare(out[:, 6 * h:6 * h + 6], lse[:, 6 * h:6 * h + 6], o_ref, l_ref)


def test_prefill_subset_of_the_524k_workload(kv_gpu):
    """The 2,048-token chunk as four ubatches of 512, over a 32,768-token prior subset, one
    KV head (6 query heads), 4,096-token KV splits: every row against single-pass softmax."""
    H, n_prior, n_chunk, ub = 1, 32768, 2048, 512
    rng, k, v, q, cache, T = _case(4004, H, n_prior, n_chunk, outliers=False)
    oc = OracleCache(k, v, "q4_0")
    for u in range(n_chunk // ub):
        rows = slice(u * ub, (u + 1) * ub)
        q_pos = np.arange(n_prior + u * ub, n_prior + (u + 1) * ub)
        out, lse = _prefill(kv_gpu, cache, 6, q[rows], q_pos, cache.page_table_np, 4096)
        o_ref, l_ref = oc.attend(q[rows], q_pos, 0, 6)
        compare(out, lse, o_ref, l_ref)


def test_prefill_largest_split(kv_gpu):
    """kv_split_tokens = 65,536 (the largest accepted): 1,024 tiles per CTA, two splits."""
    H, n_prior, n_q = 1, 70000, 16
    rng, k, v, q, cache, T = _case(1400, H, n_prior, n_q, outliers=False)
    q_pos = np.arange(n_prior, T)
    out, lse = _prefill(kv_gpu, cache, 6, q, q_pos, cache.page_table_np, 65536)
    o_ref, l_ref = OracleCache(k, v, "q4_0").attend(q, q_pos, 0, 6)
    compare(out, lse, o_ref, l_ref)


def test_prefill_bad_page_id_is_skipped_and_reported(kv_gpu):
    H, n_prior, n_q = 1, 1000, 24
    rng, k, v, q, cache, T = _case(1500, H, n_prior, n_q, outliers=False)
    plist = cache.page_table_np.copy()
    plist[0, 3] = cache.n_phys + 5
    q_pos = np.arange(n_prior, T)
    qb = torch.from_numpy(bf16_bits(q).view(np.int16)).cuda()
    out = torch.empty((n_q, 6, 256), device="cuda")
    lse = torch.empty((n_q, 6), device="cuda")
    wsb = kv_gpu.kvattn_prefill_workspace_size(cache.desc, n_q, plist.shape[1], 256)
    ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda")
    kv_gpu.kvattn_prefill_chunk(cache.desc, qb, n_q, torch.from_numpy(q_pos.astype(np.int32)).cuda(),
                                torch.from_numpy(plist).cuda(), None, None, plist.shape[1], 256, out, lse, ws, wsb)
    assert kv_gpu.kvattn_device_error() == kv_gpu.ERR_BAD_PAGE
    keys = np.arange(T)
    keys = keys[(keys < 3 * 128) | (keys >= 4 * 128)]
    o_ref, l_ref = OracleCache(k, v, "q4_0").attend(q, q_pos, 0, 6, key_idx=keys)
    compare(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


def test_prefill_empty_page_list_for_one_head(kv_gpu):
    """Head 0 lists no page: its rows see no key (o = 0, lse = -inf); head 1 is unaffected."""
    H, n_prior, n_q = 2, 600, 20
    rng, k, v, q, cache, T = _case(1600, H, n_prior, n_q, outliers=False)
    q_pos = np.arange(n_prior, T)
    nb = cache.n_blocks
    out, lse = _prefill(kv_gpu, cache, 6 * H, q, q_pos, cache.page_table_np, 256, None, [0, nb], nb)
    assert np.all(out[:, :6] == 0) and np.all(np.isneginf(lse[:, :6]))
    o_ref, l_ref = OracleCache(k, v, "q4_0").attend(q, q_pos, 1, 6)
    compare(out[:, 6:], lse[:, 6:], o_ref, l_ref)

"""GPU: LSE merge against the oracle; block summaries and selection bit-exact."""
import numpy as np
import pytest
import torch

from helpers_kv import ATOL, GpuCache, OracleCache
from oracle import attention as oatt
from oracle import select as osel
from synth import needle_blocks, normal_f32, np_rng, page_permutation, plant_needles

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_parts,rows,dim", [(1, 3, 256), (7, 40, 256), (129, 5, 64), (3, 1, 4)])
def test_merge_lse(kv_gpu, n_parts, rows, dim):
    rng = np_rng(800 + n_parts)
    o = normal_f32(rng, (n_parts, rows, dim))
    l = normal_f32(rng, (n_parts, rows)) * 5
    l[rng.random((n_parts, rows)) < 0.2] = -np.inf
    l[:, 0] = -np.inf                         # a row with no visible key anywhere
    out = torch.empty((rows, dim), device="cuda")
    lse = torch.empty((rows,), device="cuda")
    kv_gpu.kvattn_merge_lse(torch.from_numpy(o).cuda(), torch.from_numpy(l).cuda(), n_parts, rows, dim, out, lse)
    o_ref, l_ref = oatt.merge_lse(o, l)
    assert np.abs(out.cpu().numpy() - o_ref).max() <= 1e-5
    lg = lse.cpu().numpy()
    assert np.array_equal(np.isneginf(lg), np.isneginf(l_ref))
    fin = np.isfinite(l_ref)
    if fin.any():
        assert np.abs(lg[fin] - l_ref[fin]).max() <= 1e-5
    assert np.all(out.cpu().numpy()[0] == 0)


def _select_case(seed, H, n_full, tail, budget, recent, needles, group=6, k_fmt="q8_0"):
    rng = np_rng(seed)
    T = n_full * 128 + tail
    n_blocks = n_full + (1 if tail else 0)
    k = normal_f32(rng, (T, H, 256))
    v = normal_f32(rng, (T, H, 256))
    q = normal_f32(rng, (H, group, 256))
    n_cand = n_full - min(recent, n_full)
    needle_sets = []
    for h in range(H):
        nb = needle_blocks(rng, n_cand, needles)
        needle_sets.append(nb)
        kh = np.ascontiguousarray(k[:, h])
        plant_needles(kh, nb, q[h].astype(np.float64).sum(0), rng, cosine=0.9)
        k[:, h] = kh
    n_phys = H * n_blocks + 2
    v_fmt = "q4_1" if k_fmt == "q5_0" else "q4_0"
    cache = GpuCache(H, H * group, n_blocks, v_fmt, n_phys=n_phys, perm=page_permutation(rng, n_phys), k_fmt=k_fmt)
    cache.append(k, v, 0)
    return rng, k, v, q, cache, needle_sets, n_blocks, T


@pytest.mark.parametrize("seed,n_full,tail,budget,recent,k_fmt", [
    (900, 300, 37, 64, 32, "q8_0"), (901, 2048, 4, 256, 128, "q8_0"), (902, 50, 0, 80, 10, "q8_0"),
    (903, 40, 100, 8, 0, "q8_0"), (904, 300, 37, 64, 32, "q4_0"), (905, 300, 37, 64, 32, "q5_1"),
    (906, 300, 37, 64, 32, "q5_0")])
def test_summaries_and_selection_bit_exact(kv_gpu, seed, n_full, tail, budget, recent, k_fmt):
    H = 4
    rng, k, v, q, cache, needle_sets, n_blocks, T = _select_case(seed, H, n_full, tail, budget, recent,
                                                                 20 if n_full > 100 else 3, k_fmt=k_fmt)
    summ = torch.zeros((H, n_blocks, 256), device="cuda")
    kv_gpu.kvattn_block_summaries(cache.desc, cache.page_table, H, n_blocks, 0, n_full, summ)
    n_cand = n_full - min(recent, n_full)
    cap = min(budget, n_cand) + (n_blocks - n_cand)
    sel_l = torch.full((H, cap), -7, dtype=torch.int32, device="cuda")
    sel_p = torch.full((H, cap), -7, dtype=torch.int32, device="cuda")
    n_sel = torch.zeros((H,), dtype=torch.int32, device="cuda")
    wsb = kv_gpu.kvattn_select_workspace_size(H, n_blocks)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    qg = torch.from_numpy(q).cuda()
    kv_gpu.kvattn_select_blocks(summ, qg, H, 6, n_blocks, n_full, n_blocks, budget, recent, cache.page_table,
                                sel_l, sel_p, n_sel, cap, ws, wsb)
    torch.cuda.synchronize()
    oc = OracleCache(k, v, "q4_1" if k_fmt == "q5_0" else "q4_0", k_fmt)
    s_gpu = summ.cpu().numpy()
    for h in range(H):
        kc = oc.kc[: n_full * 128, h].reshape(n_full, 128, 8, 32)
        kd = oc.kd[: n_full * 128, h].reshape((n_full, 128) + oc.kd.shape[2:])  # (d, m) pairs for Q5_1
        s_ref = osel.block_summaries(kc, kd, k_fmt)
        assert np.array_equal(s_gpu[h, :n_full].view(np.uint32), s_ref.view(np.uint32))
        scores = osel.block_scores(s_ref[:n_cand], q[h])
        sel, gap = osel.select_blocks(scores, n_full, n_blocks, budget, recent)
        assert gap > 1e-9 * np.abs(scores).max(), "ambiguous seed"
        ns = int(n_sel[h])
        assert ns == len(sel)
        assert sel_l[h, :ns].cpu().numpy().tolist() == sel.tolist()
        assert sel_p[h, :ns].cpu().numpy().tolist() == cache.page_table_np[h, sel].tolist()
        if n_cand > budget:
            assert set(needle_sets[h].tolist()) <= set(sel.tolist())

"""GPU: resident-page reuse (kvattn_resident_update) against the oracle, bit-exact, over
drifting selections; the gathered pool pages against the host pages they name."""
import numpy as np
import pytest
import torch

from oracle.resident import resident_update
from synth import np_rng

pytestmark = pytest.mark.gpu


def _drift(rng, cur, n_full, k):
    keep = rng.choice(k, k - int(rng.integers(0, 7)), replace=False)
    pool = np.setdiff1d(np.arange(n_full), cur[keep])
    return np.sort(np.concatenate([cur[keep], rng.choice(pool, k - len(keep), replace=False)]))


def test_resident_update_matches_oracle(kv_gpu):
    rng = np_rng(1700)
    U, n_full, k, n_slots = 3, 300, 32, 40
    n_blocks, cap = n_full + 1, k + 1                    # + the tail block, not managed
    first_page = 1000
    sob = torch.full((U, n_blocks), -1, dtype=torch.int32, device="cuda")
    bos = torch.full((U, n_slots), -1, dtype=torch.int32, device="cuda")
    hp = torch.from_numpy(rng.permutation(U * n_blocks).astype(np.int32).reshape(U, n_blocks)).cuda()
    extra = torch.tensor([7, 8, 9], dtype=torch.int32, device="cuda")
    pl = torch.empty((U, cap), dtype=torch.int32, device="cuda")
    ch = torch.empty((U, cap), dtype=torch.int32, device="cuda")
    cd = torch.empty((U, cap), dtype=torch.int32, device="cuda")
    nc = torch.empty(U, dtype=torch.int32, device="cuda")
    o_sob = [np.full(n_blocks, -1, np.int64) for _ in range(U)]
    o_bos = [np.full(n_slots, -1, np.int64) for _ in range(U)]
    cur = [np.sort(rng.choice(n_full, k, replace=False)) for _ in range(U)]
    hpn = hp.cpu().numpy()
    for step in range(25):
        if step:
            cur = [_drift(rng, c, n_full, k) for c in cur]
        sel = np.stack([np.concatenate([c, [n_full]]) for c in cur]).astype(np.int32)
        nsel = torch.full((U,), cap, dtype=torch.int32, device="cuda")
        kv_gpu.kvattn_resident_update(torch.from_numpy(sel).cuda(), nsel, cap, U, n_blocks, n_full, sob, bos, n_slots,
                                      hp, first_page, extra, pl, ch, cd, nc)
        torch.cuda.synchronize()
        for u in range(U):
            ps, cp = resident_update(cur[u], o_sob[u], o_bos[u])
            base = first_page + u * n_slots
            assert pl[u].cpu().numpy().tolist() == (base + ps).tolist() + [int(extra[u])]
            n = int(nc[u])
            assert n == len(cp)
            assert cd[u, :n].cpu().numpy().tolist() == [base + s for _, s in cp]
            assert ch[u, :n].cpu().numpy().tolist() == [int(hpn[u, b]) for b, _ in cp]
            assert (cd[u, n:].cpu().numpy() == -1).all()
            assert sob[u].cpu().numpy().tolist() == o_sob[u].tolist()
            assert bos[u].cpu().numpy().tolist() == o_bos[u].tolist()
    assert kv_gpu.kvattn_device_error() == 0


def test_resident_pool_holds_the_selected_pages(kv_gpu):
    rng = np_rng(1701)
    U, n_full, k, n_slots, pb = 2, 120, 16, 20, 4096
    n_blocks, cap = n_full, k
    host = torch.from_numpy(rng.integers(0, 256, (U * n_blocks, pb), dtype=np.uint8)).pin_memory()
    pool = torch.zeros((U * n_slots, pb), dtype=torch.uint8, device="cuda")
    sob = torch.full((U, n_blocks), -1, dtype=torch.int32, device="cuda")
    bos = torch.full((U, n_slots), -1, dtype=torch.int32, device="cuda")
    hp = torch.arange(U * n_blocks, dtype=torch.int32, device="cuda").view(U, n_blocks)
    extra = torch.zeros(U, dtype=torch.int32, device="cuda")
    pl = torch.empty((U, cap), dtype=torch.int32, device="cuda")
    ch = torch.empty((U, cap), dtype=torch.int32, device="cuda")
    cd = torch.empty((U, cap), dtype=torch.int32, device="cuda")
    nc = torch.empty(U, dtype=torch.int32, device="cuda")
    cur = [np.sort(rng.choice(n_full, k, replace=False)) for _ in range(U)]
    copies = 0
    for step in range(8):
        if step:
            cur = [_drift(rng, c, n_full, k) for c in cur]
        sel = torch.from_numpy(np.stack(cur).astype(np.int32)).cuda()
        nsel = torch.full((U,), k, dtype=torch.int32, device="cuda")
        kv_gpu.kvattn_resident_update(sel, nsel, cap, U, n_blocks, n_full, sob, bos, n_slots, hp, 0, extra, pl, ch,
                                      cd, nc)
        kv_gpu.kvattn_gather_pages(host, pb, U * n_blocks, pool, pb, U * n_slots, pb, ch, cd, U * cap, n_ctas=4)
        torch.cuda.synchronize()
        copies += int(nc.sum())
        plc, hn, dn = pl.cpu().numpy(), host.numpy(), pool.cpu().numpy()
        for u in range(U):
            for i, b in enumerate(cur[u]):
                assert np.array_equal(dn[plc[u, i]], hn[u * n_blocks + b])
    assert copies < 8 * U * k           # pages were reused
    assert kv_gpu.kvattn_device_error() == 0


def test_too_few_slots_leaves_the_unit_unchanged(kv_gpu):
    U, n_blocks, n_slots, cap = 1, 50, 4, 6
    sob = torch.full((U, n_blocks), -1, dtype=torch.int32, device="cuda")
    bos = torch.full((U, n_slots), -1, dtype=torch.int32, device="cuda")
    hp = torch.zeros((U, n_blocks), dtype=torch.int32, device="cuda")
    extra = torch.zeros(U, dtype=torch.int32, device="cuda")
    pl, ch, cd = (torch.empty((U, cap), dtype=torch.int32, device="cuda") for _ in range(3))
    nc = torch.empty(U, dtype=torch.int32, device="cuda")
    sel = torch.arange(cap, dtype=torch.int32, device="cuda").view(U, cap)
    kv_gpu.kvattn_resident_update(sel, torch.full((U,), cap, dtype=torch.int32, device="cuda"), cap, U, n_blocks,
                                  n_blocks, sob, bos, n_slots, hp, 0, extra, pl, ch, cd, nc)
    assert kv_gpu.kvattn_device_error() == kv_gpu.ERR_INVALID_ARG
    assert int(nc[0]) == 0 and (cd.cpu().numpy() == -1).all()
    assert (sob.cpu().numpy() == -1).all() and (bos.cpu().numpy() == -1).all()


def test_decode_through_the_resident_pool(kv_gpu):
    """Full history in pinned host RAM; three steps with a drifting retrieval query select
    blocks per KV head, kvattn_resident_update maps them onto each head's slot pool, only the
    misses are gathered, and decode attends over the pool through the returned page list:
    against the oracle over the same blocks at every step."""
    from helpers_kv import GpuCache, OracleCache, compare
    from oracle import select as osel
    from synth import normal_f32

    rng = np_rng(1702)
    H, g, n_full, budget, tail = 2, 6, 64, 12, 21
    PAGE = 34816 + 18432
    T = n_full * 128 + tail
    nb = n_full + 1
    k = normal_f32(rng, (T, H, 256))
    v = normal_f32(rng, (T, H, 256))
    src = GpuCache(H, H * g, nb, "q4_0")
    src.append(k, v, 0)
    summ = torch.zeros((H, nb, 256), device="cuda")
    kv_gpu.kvattn_block_summaries(src.desc, src.page_table, H, nb, 0, n_full, summ)
    host = torch.empty((H * nb, PAGE), dtype=torch.uint8).pin_memory()
    host[:, :34816] = src.k_pool.cpu()
    host[:, 34816:] = src.v_pool.cpu()
    host_table = torch.arange(H * nb, dtype=torch.int32, device="cuda").view(H, nb)
    n_res = H * budget
    pool = torch.zeros((n_res + H, PAGE), dtype=torch.uint8, device="cuda")
    for h in range(H):
        pool[n_res + h] = host[h * nb + n_full].cuda()
    tails = torch.arange(n_res, n_res + H, dtype=torch.int32, device="cuda")
    cap = budget + 1
    sel_l, sel_p = (torch.zeros((H, cap), dtype=torch.int32, device="cuda") for _ in range(2))
    n_sel = torch.zeros((H,), dtype=torch.int32, device="cuda")
    sws = torch.zeros(kv_gpu.kvattn_select_workspace_size(H, nb), dtype=torch.uint8, device="cuda")
    sob = torch.full((H, nb), -1, dtype=torch.int32, device="cuda")
    bos = torch.full((H, budget), -1, dtype=torch.int32, device="cuda")
    pl, ch, cd = (torch.zeros((H, cap), dtype=torch.int32, device="cuda") for _ in range(3))
    nc = torch.zeros(H, dtype=torch.int32, device="cuda")
    desc = kv_gpu.make_desc(H, H * g, pool, pool.data_ptr() + 34816, n_res + H, k_page_stride=PAGE,
                            v_page_stride=PAGE)
    out = torch.empty((1, H * g, 256), device="cuda")
    lse = torch.empty((1, H * g), device="cuda")
    dws = kv_gpu.kvattn_decode_workspace_size(desc, 1, cap)
    ws = torch.zeros(max(dws, 256), dtype=torch.uint8, device="cuda")
    qpos = torch.tensor([T - 1], dtype=torch.int32, device="cuda")
    oc = OracleCache(k, v, "q4_0")
    q = normal_f32(rng, (1, H * g, 256))
    for step in range(3):
        if step:
            q = (q + 0.3 * normal_f32(rng, q.shape)).astype(np.float32)
        qd = torch.from_numpy(q).cuda()
        kv_gpu.kvattn_select_blocks(summ, qd[0].view(H, g, 256).contiguous(), H, g, nb, n_full, nb, budget, 0,
                                    host_table, sel_l, sel_p, n_sel, cap, sws, sws.numel())
        kv_gpu.kvattn_resident_update(sel_l, n_sel, cap, H, nb, n_full, sob, bos, budget, host_table, 0, tails, pl,
                                      ch, cd, nc)
        kv_gpu.kvattn_gather_pages(host, PAGE, H * nb, pool, PAGE, n_res + H, PAGE, ch, cd, H * cap, n_ctas=4)
        kv_gpu.kvattn_decode(desc, qd, 1, qpos, pl, sel_l, n_sel, cap, out, lse, ws, dws)
        torch.cuda.synchronize()
        sl = sel_l.cpu().numpy()
        for h in range(H):
            kc = oc.kc[: n_full * 128, h].reshape(n_full, 128, 8, 32)
            kd = oc.kd[: n_full * 128, h].reshape(n_full, 128, 8)
            sc = osel.block_scores(osel.block_summaries(kc, kd), q[0, h * g:(h + 1) * g])
            ref_sel, gap = osel.select_blocks(sc, n_full, nb, budget, 0)
            assert gap > 1e-9 * np.abs(sc).max()
            assert sl[h].tolist() == ref_sel.tolist()
            keys = (ref_sel[:, None] * 128 + np.arange(128)[None, :]).ravel()
            o_ref, l_ref = oc.attend(q, [T - 1], h, g, key_idx=keys[keys < T])
            compare(out[:, g * h:g * h + g].cpu().numpy(), lse[:, g * h:g * h + g].cpu().numpy(), o_ref, l_ref)
    assert kv_gpu.kvattn_device_error() == 0

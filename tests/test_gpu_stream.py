"""GPU: host-streamed pages -- cudaMemcpyAsync runs (kvattn_stream_pages), device-list
driven copies over mapped pinned memory (kvattn_gather_pages / kvattn_scatter_pages), and a
selected working set streamed from host RAM and attended over, against the oracle."""
import numpy as np
import pytest
import torch

from helpers_kv import GpuCache, OracleCache, compare
from oracle import select as osel
from synth import needle_blocks, normal_f32, np_rng, page_permutation, plant_needles

pytestmark = pytest.mark.gpu

PAGE = 34816 + 18432  # K page followed by its V page


def test_stream_pages_copies_runs(kv_gpu):
    rng = np_rng(1500)
    n_host, n_dev, pb = 40, 24, 4096
    host = torch.from_numpy(rng.integers(0, 256, (n_host, pb), dtype=np.uint8)).pin_memory()
    dev = torch.zeros((n_dev, pb), dtype=torch.uint8, device="cuda")
    hid = [3, 4, 5, 17, 30, 31, 0, 39]
    slot = [0, 1, 2, 5, 9, 10, 23, 11]
    s = torch.cuda.Stream()
    ev = torch.cuda.Event()
    n = kv_gpu.kvattn_stream_pages(host, pb, dev, pb, pb, hid, slot, copy_stream=s, done=ev)
    assert n == len(kv_gpu.kvattn_stream_plan(hid, slot)) == 5
    assert kv_gpu.kvattn_stream_wait(ev, 5000) == kv_gpu.OK
    d = dev.cpu().numpy()
    h = host.numpy()
    for a, b in zip(hid, slot):
        assert np.array_equal(d[b], h[a])
    untouched = sorted(set(range(n_dev)) - set(slot))
    assert not d[untouched].any()


def test_gather_and_scatter_pages(kv_gpu):
    rng = np_rng(1501)
    n_host, n_dev, pb = 64, 32, PAGE
    host = torch.from_numpy(rng.integers(0, 256, (n_host, pb), dtype=np.uint8)).pin_memory()
    dev = torch.zeros((n_dev, pb), dtype=torch.uint8, device="cuda")
    hid = torch.tensor([7, 63, 0, 12, 12, 40], dtype=torch.int32, device="cuda")
    slot = torch.tensor([0, 31, 5, 6, -1, 2], dtype=torch.int32, device="cuda")
    kv_gpu.kvattn_gather_pages(host, pb, n_host, dev, pb, n_dev, pb, hid, slot, 6, n_ctas=3)
    torch.cuda.synchronize()
    d, h = dev.cpu().numpy(), host.numpy()
    for a, b in [(7, 0), (63, 31), (0, 5), (12, 6), (40, 2)]:
        assert np.array_equal(d[b], h[a])
    # device -> host: scatter slot 31 to host page 1
    kv_gpu.kvattn_scatter_pages(host, pb, n_host, dev, pb, n_dev, pb, torch.tensor([1], dtype=torch.int32,
                                device="cuda"), torch.tensor([31], dtype=torch.int32, device="cuda"), 1)
    torch.cuda.synchronize()
    assert np.array_equal(host.numpy()[1], h[63])
    assert kv_gpu.kvattn_device_error() == 0
    # an id out of range is skipped and reported
    kv_gpu.kvattn_gather_pages(host, pb, n_host, dev, pb, n_dev, pb, torch.tensor([64], dtype=torch.int32,
                               device="cuda"), torch.tensor([0], dtype=torch.int32, device="cuda"), 1)
    assert kv_gpu.kvattn_device_error() == kv_gpu.ERR_BAD_PAGE


def test_gather_refuses_pageable_host_memory(kv_gpu):
    host = torch.zeros((4, 4096), dtype=torch.uint8)          # not pinned
    dev = torch.zeros((4, 4096), dtype=torch.uint8, device="cuda")
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(kv_gpu.KVAttnError) as e:
        kv_gpu.kvattn_gather_pages(host, 4096, 4, dev, 4096, 4, 4096, ids, ids, 1)
    assert e.value.status == kv_gpu.ERR_INVALID_ARG


def test_streamed_working_set_decode(kv_gpu):
    """Full history in pinned host RAM; per KV head the retrieval query selects `budget`
    blocks, the copy kernel brings them (and the tail page stays resident) into device slots,
    and decode attends over them: against the oracle over the same blocks."""
    rng = np_rng(1502)
    H, g, n_full, budget = 4, 6, 96, 24
    tail = 37
    T = n_full * 128 + tail
    nb = n_full + 1
    k = normal_f32(rng, (T, H, 256))
    v = normal_f32(rng, (T, H, 256))
    q = normal_f32(rng, (1, H * g, 256))
    needles = []
    for h in range(H):
        nbk = needle_blocks(rng, n_full, 6)
        needles.append(nbk)
        kh = np.ascontiguousarray(k[:, h])
        plant_needles(kh, nbk, q[0, h * g:(h + 1) * g].astype(np.float64).sum(0), rng, cosine=0.9)
        k[:, h] = kh
    # build the cache on the device (interleaved K|V pages), then move it to pinned host RAM
    src = GpuCache(H, H * g, nb, "q4_0")
    src.append(k, v, 0)
    summ = torch.zeros((H, nb, 256), device="cuda")
    kv_gpu.kvattn_block_summaries(src.desc, src.page_table, H, nb, 0, n_full, summ)
    host = torch.empty((H * nb, PAGE), dtype=torch.uint8).pin_memory()
    host[:, :34816] = src.k_pool.cpu()
    host[:, 34816:] = src.v_pool.cpu()
    host_table = torch.arange(H * nb, dtype=torch.int32, device="cuda").view(H, nb)
    # device slots: budget streamed slots per head + one resident tail slot per head
    n_slots = H * budget + H
    slots = torch.zeros((n_slots, PAGE), dtype=torch.uint8, device="cuda")
    for h in range(H):
        slots[H * budget + h] = host[h * nb + n_full].cuda()
    cap = budget + 1
    sel_l = torch.zeros((H, cap), dtype=torch.int32, device="cuda")
    sel_p = torch.zeros((H, cap), dtype=torch.int32, device="cuda")
    n_sel = torch.zeros((H,), dtype=torch.int32, device="cuda")
    wsb = kv_gpu.kvattn_select_workspace_size(H, nb)
    sws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    qd = torch.from_numpy(q).cuda()
    kv_gpu.kvattn_select_blocks(summ, qd[0].view(H, g, 256).contiguous(), H, g, nb, n_full, nb, budget, 0,
                                host_table, sel_l, sel_p, n_sel, cap, sws, wsb)
    dst = torch.tensor([[h * budget + i if i < budget else -1 for i in range(cap)] for h in range(H)],
                       dtype=torch.int32, device="cuda")
    kv_gpu.kvattn_gather_pages(host, PAGE, H * nb, slots, PAGE, n_slots, PAGE, sel_p, dst, H * cap, n_ctas=8)
    plist = torch.tensor([[h * budget + i if i < budget else H * budget + h for i in range(cap)] for h in range(H)],
                         dtype=torch.int32, device="cuda")
    desc = kv_gpu.make_desc(H, H * g, slots, slots.data_ptr() + 34816, n_slots, k_page_stride=PAGE,
                            v_page_stride=PAGE)
    out = torch.empty((1, H * g, 256), device="cuda")
    lse = torch.empty((1, H * g), device="cuda")
    dws = kv_gpu.kvattn_decode_workspace_size(desc, 1, cap)
    ws = torch.zeros(max(dws, 256), dtype=torch.uint8, device="cuda")
    qpos = torch.tensor([T - 1], dtype=torch.int32, device="cuda")
    kv_gpu.kvattn_decode(desc, qd, 1, qpos, plist, sel_l, n_sel, cap, out, lse, ws, dws)
    torch.cuda.synchronize()
    oc = OracleCache(k, v, "q4_0")
    sl = sel_l.cpu().numpy()
    for h in range(H):
        kc = oc.kc[: n_full * 128, h].reshape(n_full, 128, 8, 32)
        kd = oc.kd[: n_full * 128, h].reshape(n_full, 128, 8)
        sc = osel.block_scores(osel.block_summaries(kc, kd), q[0, h * g:(h + 1) * g])
        ref_sel, gap = osel.select_blocks(sc, n_full, nb, budget, 0)
        assert gap > 1e-9 * np.abs(sc).max()
        assert sl[h].tolist() == ref_sel.tolist()
        assert set(needles[h].tolist()) <= set(ref_sel.tolist())
        keys = (ref_sel[:, None] * 128 + np.arange(128)[None, :]).ravel()
        keys = keys[keys < T]
        o_ref, l_ref = oc.attend(q, [T - 1], h, g, key_idx=keys)
        compare(out[:, g * h:g * h + g].cpu().numpy(), lse[:, g * h:g * h + g].cpu().numpy(), o_ref, l_ref)


def test_stream_wait_times_out_then_completes(kv_gpu):
    """An event behind a bounded busy kernel (at least 0.75 s) has not fired after 20 ms:
    the wait returns TIMEOUT and the context stays usable; a longer wait then succeeds."""
    s = torch.cuda.Stream()
    ev = torch.cuda.Event()
    with torch.cuda.stream(s):
        torch.cuda._sleep(int(1.5e9))          # clock cycles; ends by itself
        ev.record(s)
    assert kv_gpu.kvattn_stream_wait(ev, 20) == kv_gpu.ERR_TIMEOUT
    assert kv_gpu.kvattn_stream_wait(ev, 10000) == kv_gpu.OK
    assert kv_gpu.kvattn_device_error() == 0

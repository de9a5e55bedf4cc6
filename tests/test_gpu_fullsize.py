"""GPU parity at the benchmark's full sizes, in the launch configuration the benchmark times.

Each test builds one layer of a benchmark workload through the benchmark's own classes (same
context length, head counts, page table, split plan and launch sequence as every timed
layer), runs that layer once, and checks outputs against the oracle:

* decode, 131,072 tokens (every supported K / V format pair): every
  output row of the layer, plus page bytes of sampled blocks bit-exact;
* MTP verify, 262,144 tokens + 4: the selection bit-exact (needles included) and the 4 x 24
  rows over the selected blocks, for two sampled KV heads;
* chunked prefill, 524,288 prior tokens + the 2,048-token chunk: 64 seeded (token, query head)
  rows over the full context;
* the host-streamed generation over 524,288 prompt tokens: 512 advancing steps, selection and
  decode rows of two KV heads at steps 0, 255 and 511, and the host bytes of every generated
  token's pages.

The oracle's inputs are the same seeded draws (made on the device by torch's generator and
copied to the host) with the oracle's own quantisation; nothing the CUDA library computes
reaches the oracle."""
import numpy as np
import pytest
import torch

import bench
from helpers_kv import OracleCache, compare
from oracle import attention as oatt
from oracle import select as osel
from synth import np_rng, workload_layer_kv

pytestmark = [pytest.mark.gpu]

DEV = "cuda"


def _head(x, h):
    return x[:, h].contiguous().cpu().numpy()


def _oracle_unit(k, v, h, v_fmt, k_tail=None, v_tail=None, k_fmt="q8_0"):
    """OracleCache of KV head h: the workload's draws, then the appended tokens."""
    kh, vh = _head(k, h), _head(v, h)
    if k_tail is not None:
        kh = np.concatenate([kh, k_tail[:, h].cpu().numpy()], 0)
        vh = np.concatenate([vh, v_tail[:, h].cpu().numpy()], 0)
    return OracleCache(kh[:, None], vh[:, None], v_fmt, k_fmt)


@pytest.mark.parametrize("wname", ["decode131k", "decode131k_q8q8", "decode131k_q4q4", "decode131k_q4q8",
                                   "decode131k_q51q4", "decode131k_q51q8", "decode131k_q50q41"])
def test_decode_full_context(kv_gpu, wname):
    b = bench.DecodeBench(kv_gpu, wname, torch.device(DEV), layers=1)
    b.layer(0)
    torch.cuda.synchronize()
    assert kv_gpu.kvattn_device_error() == 0
    w, ctx, g = b.w, b.ctx, b.w.group
    out, lse = b.out[0].cpu().numpy(), b.lse[0].cpu().numpy()
    k, v, _ = workload_layer_kv(w, 0, ctx, DEV)
    # the step's new token overwrites the last position
    k[ctx - 1] = b.k_new[0, 0]
    v[ctx - 1] = b.v_new[0, 0]
    q = b.q[0].cpu().numpy()
    pt = b.cache.page_table[0].cpu().numpy()
    rng = np_rng(7100)
    for h in range(w.kv_heads):
        oc = _oracle_unit(k, v, h, w.v_fmt, k_fmt=w.k_fmt)
        for blk in [0, b.nb - 1] + rng.choice(b.nb, 4, replace=False).tolist():
            phys = int(pt[h, blk])
            assert np.array_equal(b.cache.k_pool[phys].cpu().numpy(), oc.page_bytes(0, blk, "k"))
            assert np.array_equal(b.cache.v_pool[phys].cpu().numpy(), oc.page_bytes(0, blk, "v"))
        o_ref, l_ref = oc.attend(q[:, h * g:(h + 1) * g], [ctx - 1], 0, g)
        compare(out[:, h * g:(h + 1) * g], lse[:, h * g:(h + 1) * g], o_ref, l_ref)


def test_decode_repeated_launches_bit_identical(kv_gpu):
    """Hundreds of back-to-back launches of the benchmark's decode layer: the stage ring of
    every CTA is exercised under varying copy completion orders; every launch must give the
    same bits and no wait may expire."""
    b = bench.DecodeBench(kv_gpu, "decode131k", torch.device(DEV), layers=1)
    b.layer(0)
    torch.cuda.synchronize()
    ref_o, ref_l = b.out[0].clone(), b.lse[0].clone()
    for _ in range(300):
        b.layer(0)
    torch.cuda.synchronize()
    assert kv_gpu.kvattn_device_error() == 0
    assert torch.equal(b.out[0], ref_o) and torch.equal(b.lse[0], ref_l)


def _selected_keys(sel, T):
    keys = (np.asarray(sel)[:, None] * 128 + np.arange(128)[None, :]).ravel()
    return keys[keys < T]


def test_verify_full_context(kv_gpu):
    b = bench.VerifyBench(kv_gpu, torch.device(DEV), layers=1)
    b.layer(0)
    torch.cuda.synchronize()
    assert kv_gpu.kvattn_device_error() == 0
    w, g = b.w, b.w.group
    ctx = w.context
    k, v, needles = workload_layer_kv(w, 0, ctx, DEV, b.q[0])
    q = b.q[0].cpu().numpy()
    out, lse = b.out[0].cpu().numpy(), b.lse[0].cpu().numpy()
    sel_l, n_sel = b.sel_l[0].cpu().numpy(), b.n_sel[0].cpu().numpy()
    for h in (0, w.kv_heads - 1):
        oc = _oracle_unit(k, v, h, w.v_fmt, b.k_new[0], b.v_new[0])
        T = ctx + w.n_q
        kc = oc.kc[: b.n_full * 128, 0].reshape(b.n_full, 128, 8, 32)
        kd = oc.kd[: b.n_full * 128, 0].reshape(b.n_full, 128, 8)
        sc = osel.block_scores(osel.block_summaries(kc, kd), q[-1, h * g:(h + 1) * g])
        ref_sel, gap = osel.select_blocks(sc, b.n_full, b.nb, w.budget_blocks, w.recent_blocks)
        assert gap > 1e-9 * np.abs(sc).max()
        assert sel_l[h, : n_sel[h]].tolist() == ref_sel.tolist()
        assert set(needles[h].tolist()) <= set(ref_sel.tolist())
        o_ref, l_ref = oc.attend(q[:, h * g:(h + 1) * g], list(range(ctx, T)), 0, g,
                                 key_idx=_selected_keys(ref_sel, T))
        compare(out[:, h * g:(h + 1) * g], lse[:, h * g:(h + 1) * g], o_ref, l_ref)


@pytest.mark.parametrize("wname,f16", [("prefill524k", False), ("prefill524k_q4q4", False),
                                       ("prefill524k_q51q4", False), ("prefill524k_q50q41", False),
                                       ("prefill524k_q8q8", False), ("prefill524k", True)])
def test_prefill_full_context_sampled_rows(kv_gpu, wname, f16):
    """One layer of the 524,288-key prefill as the bench runs it (the f16 case through
    kvattn_prefill_chunk_f16): 64 sampled rows of two KV heads against the oracle."""
    b = bench.PrefillBench(kv_gpu, torch.device(DEV), layers=1, wname=wname, f16=f16)
    b.layer(0)
    torch.cuda.synchronize()
    assert kv_gpu.kvattn_device_error() == 0
    w, g = b.w, b.w.group
    ctx, T = w.context, b.total
    rng = np_rng(7200)
    heads = np.sort(rng.choice(w.kv_heads, 2, replace=False))
    k, v, _ = workload_layer_kv(w, 0, ctx, DEV)
    q = b.q[0].float().cpu().numpy()                   # bf16 values, exact in fp32
    out, lse = b.out[0].cpu().numpy(), b.lse[0].cpu().numpy()
    for h in heads:
        oc = _oracle_unit(k, v, int(h), w.v_fmt, b.k_new[0], b.v_new[0], k_fmt=w.k_fmt)
        t = np.sort(rng.choice(w.n_q, 32, replace=False))
        j = h * g + rng.integers(0, g, 32)
        rows = q[t, j]
        o_ref, l_ref = oatt.attend(rows, oc.khat(0), oc.vhat(0), np.arange(T), ctx + t, 1.0 / 16.0)
        compare(out[t, j], lse[t, j], o_ref, l_ref)


def test_stream_full_context(kv_gpu):
    """The host-streamed generation at full size (one layer): 512 decode steps whose position
    advances from 524,288; steps 0, 255 and 511 are checked against the oracle (selection
    bit-exact, decode rows within the tolerance) and, after the generation, the host bytes of
    every appended token's pages bit-exact."""
    b = bench.StreamBench(kv_gpu, torch.device(DEV), layers=1)
    w, g = b.w, b.w.group
    ctx, S = w.context, w.steps
    checks = {0: None, 255: None, 511: None}
    for t in range(S):
        b.step(True)
        if t in checks:
            torch.cuda.synchronize()
            checks[t] = (b.out[0].cpu().numpy(), b.lse[0].cpu().numpy(), b.sel_l[0].cpu().numpy(),
                         b.n_sel[0].cpu().numpy())
    torch.cuda.synchronize()
    assert kv_gpu.kvattn_device_error() == 0
    k, v, _ = workload_layer_kv(w, 0, ctx, DEV)
    k_gen, v_gen = b.k_all[:, 0, 0], b.v_all[:, 0, 0]            # [S][H][256]
    q_all = b.q_all[:, 0, 0].cpu().numpy()                        # [S][Hq][256]
    host = b.host.numpy()
    for h in (1, 2):
        oc = _oracle_unit(k, v, h, w.v_fmt, k_gen, v_gen)
        kc = oc.kc[: b.n_full * 128, 0].reshape(b.n_full, 128, 8, 32)
        kd = oc.kd[: b.n_full * 128, 0].reshape(b.n_full, 128, 8)
        summ = osel.block_summaries(kc, kd)
        for t, (out, lse, sel_l, n_sel) in checks.items():
            T = ctx + t + 1
            n_total = b.n_full + t // 128 + 1
            sc = osel.block_scores(summ, q_all[t, h * g:(h + 1) * g])
            ref_sel, gap = osel.select_blocks(sc, b.n_full, n_total, w.budget_blocks, 0)
            assert gap > 1e-9 * np.abs(sc).max()
            assert sel_l[h, : n_sel[h]].tolist() == ref_sel.tolist(), t
            o_ref, l_ref = oc.attend(q_all[t:t + 1, h * g:(h + 1) * g], [ctx + t], 0, g,
                                     key_idx=_selected_keys(ref_sel, T))
            compare(out[:, h * g:(h + 1) * g], lse[:, h * g:(h + 1) * g], o_ref, l_ref)
        # every generated token's page in host RAM, bit-exact (the pages the generation filled)
        for kk in range(b.n_tail):
            blk = b.n_full + kk
            page = host[int(b.tail_hosts[0, h, kk])]
            assert np.array_equal(page[:34816], oc.page_bytes(0, blk, "k")), (h, kk, "k")
            assert np.array_equal(page[34816:], oc.page_bytes(0, blk, "v")), (h, kk, "v")

"""Host logic of the multi-GPU decode split on CPU: two gloo ranks (127.0.0.1).

* the unit and page ranges partition their items exactly (every item once, sizes within one);
* the sequence split: each rank attends over its page range of every head (the oracle stands
  in for the CUDA decode on CPU), the (o, lse) partials are all-gathered with the same
  collective the GPU path uses, and their log-sum-exp merge equals single-pass attention over
  the whole list (to fp64 rounding)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from quantized_paged_kv_q4_b200 import shard


@pytest.mark.parametrize("n,world", [(64, 2), (64, 3), (5, 8), (0, 4), (1025, 7)])
def test_balanced_ranges_partition(n, world):
    seen = []
    sizes = []
    for r in range(world):
        a, b = shard.balanced_range(n, world, r)
        seen.extend(range(a, b))
        sizes.append(b - a)
    assert seen == list(range(n))
    assert max(sizes) - min(sizes) <= 1


def test_unit_ranges_cover_all_units_once():
    units = []
    for r in range(3):
        units += shard.unit_range(16, 4, 3, r)
    assert units == [(l, h) for l in range(16) for h in range(4)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    from oracle import attention as oatt
    from synth import normal_f32, np_rng

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        rng = np_rng(7700)                        # the same draws on every rank
        n_pages, rows, D = 9, 6, 256
        k = normal_f32(rng, (n_pages * 128, D)).astype(np.float64)
        v = normal_f32(rng, (n_pages * 128, D)).astype(np.float64)
        q = normal_f32(rng, (rows, D)).astype(np.float64)
        order = rng.permutation(n_pages)          # the page list, in any order
        a, b = shard.page_range(n_pages, world, rank)
        keys = (order[a:b][:, None] * 128 + np.arange(128)[None, :]).ravel()
        pos = np.arange(n_pages * 128)
        qpos = np.full(rows, n_pages * 128 - 1)
        o_r, l_r = oatt.attend(q, k[keys], v[keys], pos[keys], qpos, 1.0 / 16.0)
        o_all, l_all = shard.gather_partials(torch.from_numpy(o_r), torch.from_numpy(l_r))
        o, l = oatt.merge_lse(o_all.numpy(), l_all.numpy())
        o_ref, l_ref = oatt.attend(q, k, v, pos, qpos, 1.0 / 16.0)
        out.put((rank, float(np.abs(o - o_ref).max()), float(np.abs(l - l_ref).max()), (a, b)))
    finally:
        dist.destroy_process_group()


def test_sequence_split_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[3] for r in res] == [(0, 5), (5, 9)]
    for _, eo, el, _ in res:
        assert eo < 1e-12 and el < 1e-12

"""Multi-process host logic of the benchmark on CPU: world size 2 over gloo (127.0.0.1).

Each rank runs an independent workload (weak scaling, no data-path collective); the
benchmark only needs a barrier, the max over ranks of the per-step time, the whole-job
throughput, and the rule that only rank 0 runs and prints the reference arm."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = [2.0, 3.5][rank]                       # per-rank device time per step
        ms_max = bench.max_over_ranks(ms, world)
        value = bench.job_throughput(1000.0, world, ms_max)

        class Args:
            steps, warmup, gpus = 1, 0, world

        # the reference arm: rank 0 alone runs it; other ranks return at once without work
        ran = False
        if rank != 0:
            bench.reference_arm(Args, world, rank)
        else:
            ran = True
        bench.barrier(world)
        out.put((rank, ms_max, value, ran))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
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
    assert [r[1] for r in res] == [3.5, 3.5]                     # both ranks see the max
    assert res[0][2] == pytest.approx(1000.0 * 2 / 3.5e-3)        # all ranks' units / slowest time
    assert res[0][3] is True and res[1][3] is False

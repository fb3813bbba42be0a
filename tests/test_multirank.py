"""The multi-rank host path of bench.py on CPU (gloo, world size 2): barrier,
max-over-ranks timing and the whole-job aggregate.  The data path needs no
collective (each rank runs its own replica of the workload), so these are the
only cross-rank steps."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.rank_barrier()
        local_ms = 10.0 * (rank + 1)          # rank 1 is the slow one
        ms_max = bench.reduce_max(local_ms)
        gbs = bench.aggregate_gbs(bench.STEP_BYTES, 100, world, ms_max)
        q.put((rank, ms_max, gbs))
        bench.rank_barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_time_and_sum_the_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms_max, gbs in res:
        assert ms_max == 20.0
        assert gbs == pytest.approx(bench_step_bytes() * 100 * 2 / 20e-3 / 1e9)


def bench_step_bytes():
    import bench
    return bench.STEP_BYTES


def test_single_rank_helpers_are_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5
    bench.rank_barrier()
    assert bench.STEP_BYTES == 75497472

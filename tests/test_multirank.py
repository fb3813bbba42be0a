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


# ----------------------------------------------------------------------------- the row split of W (N-split)
#
# Each rank takes a contiguous range of W's rows (packed codes, scales and
# biases sliced together: groups run along K inside one row, so the slices are
# themselves valid quantized matrices), computes its columns of y, and one
# all-gather assembles y.  On CPU the oracle computes each rank's columns (it
# is the checker here); the split, the slicing and the collective are the
# library's own host code (weight_only_group_b200.shard).

def _split_worker(rank, world, port, q, M, N, K, G, bits):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import numpy as np

    import oracle
    import synth
    from weight_only_group_b200 import shard
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.weights(N, K, 3100 + N, True)
        p, s, b = oracle.quantize(w, G, bits)
        xb = synth.bf16_bits(synth.activations(M, K, 3200 + N))
        pt, st, bt = torch.from_numpy(p.view(np.int32)), torch.from_numpy(s.view(np.int16)), torch.from_numpy(b.view(np.int16))
        pl, sl, bl, n0, n1 = shard.shard_rows(pt, st, bt, world, rank)
        assert n1 == n0 or pl.data_ptr() == pt[n0:].data_ptr()  # a view, not a copy
        if n1 > n0:
            y_local = oracle.matmul(xb, pl.numpy().view(np.uint32), sl.numpy().view(np.uint16),
                                    bl.numpy().view(np.uint16), G, bits)
        else:
            y_local = np.zeros((M, 0))
        y = shard.all_gather_columns(torch.from_numpy(y_local), N)
        y_full = oracle.matmul(xb, p, s, b, G, bits)
        q.put((rank, n0, n1, bool(np.array_equal(y.numpy(), y_full))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M,N,K,G,bits", [(3, 256, 512, 64, 4), (2, 200, 384, 128, 3), (1, 8, 256, 32, 2)])
def test_row_split_over_two_ranks_reassembles_the_unsplit_product(M, N, K, G, bits):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, q, M, N, K, G, bits)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[0] for r in res] == [0, 1]
    assert res[0][1] == 0 and res[0][2] == res[1][1] and res[1][2] == N  # contiguous, covers [0, N)
    assert all(r[3] for r in res), res  # bit-equal to the unsplit product on every rank


def test_row_range_partitions_every_n():
    from weight_only_group_b200 import shard
    for N in (1, 15, 16, 17, 100, 4096, 14336, 28672):
        for world in (1, 2, 3, 4, 8):
            rs = [shard.row_range(N, world, r) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == N
            assert all(rs[i][1] == rs[i + 1][0] for i in range(world - 1))
            assert all(a % shard.ROW_ALIGN == 0 for a, _ in rs)
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= shard.ROW_ALIGN
    with pytest.raises(ValueError):
        shard.row_range(10, 2, 2)

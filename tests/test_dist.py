"""The multi-rank bench logic (weak scaling, max-over-ranks time, whole-job
work) on two gloo ranks on the CPU: no GPU and no data-path collective."""
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # Rank r "ran" its batch in (1 + r) seconds doing 10 units of work.
        value, t = bench.aggregate(10.0e12, 1.0 + rank, world)
        q.put((rank, value, t, bench.max_over_ranks(3.0 * (rank + 1), world),
               bench.sum_over_ranks(rank + 1, world)))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, t, mx, sm in out:
        assert t == 2.0            # the slower rank's time
        assert value == 10.0       # 20e12 FLOPs over 2 s = 10 TFLOP/s
        assert mx == 6.0 and sm == 3.0


def _shard_worker(rank, world, port, q):
    import numpy as np
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import lrgen
        import oracle
        rows = 3
        X = bench.rank_rows(rank, rows=rows)            # this rank's rows of the batch
        p = lrgen.lowrank_problem(1, bench.K, 16, 32, seed=3)  # factors, the same on every rank
        Y = oracle.lr_linear(X, p["A"], p["B"], None)
        parts = [torch.zeros((rows, 32), dtype=torch.float64) for _ in range(world)]
        dist.all_gather(parts, torch.from_numpy(Y))
        xs = [torch.zeros((rows, bench.K), dtype=torch.int32) for _ in range(world)]
        dist.all_gather(xs, torch.from_numpy(X.astype(np.int32)))
        if rank == 0:
            whole = bench.rank_rows(0, rows=rows * world)  # the job's batch drawn whole
            Yw = oracle.lr_linear(whole, p["A"], p["B"], None)
            q.put((np.array_equal(np.concatenate([x.numpy() for x in xs]).astype(np.uint16), whole),
                   np.array_equal(np.concatenate([t.numpy() for t in parts]), Yw)))
    finally:
        dist.destroy_process_group()


def test_two_rank_row_shards_match_the_whole_batch():
    """Each rank draws its own rows of the job's batch (bench.rank_rows) and
    computes them with the factors every rank holds; gathered, the rows and
    the outputs are exactly the whole batch's (checked with the oracle on
    the CPU; the GPU kernels are row-independent in the same way)."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    same_rows, same_out = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert same_rows and same_out

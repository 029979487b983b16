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

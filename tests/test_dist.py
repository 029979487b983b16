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


def _rsplit_worker(rank, world, port, q):
    import numpy as np
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import lrgen
        import oracle
        from rank_linear_layers_b200 import rsplit
        M, K, r, N = 5, 96, 73, 40
        p = lrgen.lowrank_problem(M, K, r, N, seed=11, bias=True)
        r0, r1 = rsplit.rsplit_bounds(r, world, rank)

        def ref_partial(X, A, B, bias):
            # The oracle on this rank's slice (fp64 -> fp32), bias as given.
            return torch.from_numpy(oracle.lr_linear(X, A, B, bias).astype(np.float32))

        Y = rsplit.lr_linear_rsplit(p["X"], np.ascontiguousarray(p["A"][:, r0:r1]),
                                    np.ascontiguousarray(p["B"][r0:r1, :]), p["bias"],
                                    local_product=ref_partial)
        whole = oracle.lr_linear(p["X"], p["A"], p["B"], p["bias"])
        err = float(np.max(np.abs(Y.numpy().astype(np.float64) - whole)))
        q.put((rank, r0, r1, err, float(np.sqrt(np.mean(whole ** 2)))))
    finally:
        dist.destroy_process_group()


def test_two_rank_rsplit_sums_the_slices():
    """r split over 2 gloo ranks: each rank's slice of A and B (16-aligned
    bounds), one all-reduce; every rank ends with the whole layer's output
    (bias added once), up to the fp32 rounding of the partials."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rsplit_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, a0, a1, e0, rms), (_, b0, b1, e1, _) = out
    assert (a0, a1, b0, b1) == (0, 32, 32, 73)  # five 16-wide pieces: 2 + 3
    assert max(e0, e1) <= 1e-6 * rms


def test_rsplit_bounds():
    from rank_linear_layers_b200.rsplit import rsplit_bounds
    for r in (0, 1, 15, 16, 17, 1741, 2867, 4096):
        for world in (1, 2, 3, 4, 8):
            spans = [rsplit_bounds(r, world, i) for i in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == r
            for (x0, x1), (y0, y1) in zip(spans, spans[1:]):
                assert x1 == y0 and x0 <= x1
            assert all(x0 % 16 == 0 for x0, _ in spans)

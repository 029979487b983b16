"""Prefill calls queued on one stream without synchronising in between.

A prefill call whose operand rows are not 32-byte aligned first copies that
operand to a 128-byte pitch, and the copy may start while the library's
previous prefill launch on the stream still runs (programmatic dependent
launch).  Queued calls must give the bits of the same calls run one at a
time (split K off, so every sum is formed in a fixed order), also when a
call's A is the output of the call just before it, which the copy must not
read early.  One call of each sequence is checked against the oracle too.
"""
import numpy as np
import pytest

import lrgen
import oracle
from helpers import compare, f32_host, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lr():
    import torch
    import rank_linear_layers_b200 as lr
    lr.set_path(lr.PATH_AUTO)
    lr.set_split_k(False)
    try:
        yield lr
    finally:
        lr.set_split_k(True)
        lr.set_early_copy(True)
        torch.cuda.synchronize()


def one_at_a_time(lr, calls):
    import torch
    out = []
    for X, A, B in calls:
        out.append(lr.lr_linear(X, A, B))
        torch.cuda.synchronize()
    assert lr.last_device_status() == lr.LR_OK
    return out


def queued(lr, calls):
    import torch
    out = [lr.lr_linear(X, A, B) for X, A, B in calls]
    torch.cuda.synchronize()
    assert lr.last_device_status() == lr.LR_OK
    return out


def sampled_rows(M, seed):
    rows = np.random.default_rng(seed).choice(M, 48, replace=False)
    return np.concatenate([rows, [0, 127, 128, M - 1]])


def test_queued_prefill_calls_match_one_at_a_time(lr):
    """Three prefill calls with r = 333 (A has 666-byte rows) and a CTA on
    every SM, queued back to back, twice over."""
    import torch
    M, K, r, N = 2048, 1024, 333, 4096
    probs = [lrgen.lowrank_problem(M, K, r, N, seed=40 + i) for i in range(3)]
    calls = [(to_dev(q["X"]), to_dev(q["A"]), to_dev(q["B"])) for q in probs]
    ref = one_at_a_time(lr, calls)
    rows = sampled_rows(M, 1)
    q = probs[1]
    Y32 = lr.lr_linear_f32(*calls[1])
    torch.cuda.synchronize()
    compare(f32_host(Y32)[rows], oracle.lr_linear(q["X"], q["A"], q["B"], None, rows=rows),
            "r=333 sampled rows (fp32 output of the same call)")
    for rep in range(2):
        got = queued(lr, calls)
        for i, (g, e) in enumerate(zip(got, ref)):
            assert torch.equal(g, e), f"pass {rep}: queued call {i} differs from one at a time"


def test_queued_call_reads_previous_output(lr):
    """Call 2's A is call 1's Y ([4096, 1000]: 2000-byte rows, so it is
    copied first); call 1 has a CTA on every SM.  The copy must wait for
    call 1's launch to finish."""
    import torch
    p1 = lrgen.lowrank_problem(4096, 512, 200, 1000, seed=50)
    p2 = lrgen.lowrank_problem(256, 4096, 1000, 512, seed=51)  # A replaced by call 1's Y
    X1, A1, B1 = to_dev(p1["X"]), to_dev(p1["A"]), to_dev(p1["B"])
    X2, B2 = to_dev(p2["X"]), to_dev(p2["B"])
    Y1s = lr.lr_linear(X1, A1, B1)
    torch.cuda.synchronize()
    Y2s = lr.lr_linear(X2, Y1s, B2)
    torch.cuda.synchronize()
    assert lr.last_device_status() == lr.LR_OK
    rows = sampled_rows(4096, 2)
    Y32 = lr.lr_linear_f32(X1, A1, B1)
    torch.cuda.synchronize()
    compare(f32_host(Y32)[rows], oracle.lr_linear(p1["X"], p1["A"], p1["B"], None, rows=rows),
            "call 1 sampled rows (fp32 output of the same call)")
    for rep in range(3):
        Y1 = lr.lr_linear(X1, A1, B1)
        Y2 = lr.lr_linear(X2, Y1, B2)
        torch.cuda.synchronize()
        assert lr.last_device_status() == lr.LR_OK
        assert torch.equal(Y1, Y1s), f"pass {rep}: call 1 differs"
        assert torch.equal(Y2, Y2s), f"pass {rep}: call 2 read call 1's Y too early"


def test_early_copy_off_gives_the_same_bits(lr):
    """With the early copy off every call's first copy waits for all earlier
    work on the stream; the arithmetic, and so the result, is unchanged."""
    import torch
    M, K, r, N = 2048, 1024, 333, 4096
    probs = [lrgen.lowrank_problem(M, K, r, N, seed=60 + i) for i in range(2)]
    calls = [(to_dev(q["X"]), to_dev(q["A"]), to_dev(q["B"])) for q in probs]
    on = queued(lr, calls)
    lr.set_early_copy(False)
    try:
        off = queued(lr, calls)
    finally:
        lr.set_early_copy(True)
    for i, (a, b) in enumerate(zip(on, off)):
        assert torch.equal(a, b), f"call {i}: early copy off changed the result"

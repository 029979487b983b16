"""Failure detection without a GPU fault: every device-side wait of the
prefill kernels is bounded.  The copy thread is told to withhold the first
pipeline stage (a barrier nothing arrives on), and the wait limit is set to
5 ms: the tensor-core thread's wait runs out, the kernel records
LR_ERR_TIMEOUT in the device status word, lets its in-flight copies land,
frees its tensor memory and returns.  The host reads the status, and the
context stays usable: the next call is correct.  Nothing here traps,
asserts on the device or hangs."""
import pytest

import lrgen
import oracle
from helpers import compare, to_dev, to_f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_recovers():
    import torch
    import rank_linear_layers_b200 as lr
    p = lrgen.lowrank_problem(512, 1024, 256, 512, seed=9)
    X, A, B = to_dev(p["X"]), to_dev(p["A"]), to_dev(p["B"])
    assert lr.last_device_status() == lr.LR_OK
    lr.set_path(lr.PATH_PREFILL)
    lr.set_wait_limit_ns(5_000_000)
    lr.set_withhold_first_stage(True)
    try:
        lr.lr_linear(X, A, B)
        torch.cuda.synchronize()
        assert lr.last_device_status() == lr.LR_ERR_TIMEOUT
    finally:
        lr.set_withhold_first_stage(False)
        lr.set_wait_limit_ns(0)
        lr.set_path(lr.PATH_AUTO)
    # Cleared by the read above; a normal call afterwards is right.
    assert lr.last_device_status() == lr.LR_OK
    Y = lr.lr_linear(X, A, B)
    torch.cuda.synchronize()
    assert lr.last_device_status() == lr.LR_OK
    compare(to_f64(Y), oracle.lr_linear(p["X"], p["A"], p["B"]), "after timeout")

"""lr_linear_decode_static: the decode path for callers that cannot let a
library allocate device memory (a serving loop that cannot afford the device
synchronisation cudaMalloc/cudaFree cause, or a host whose own pool owns all
device memory).  Its scratch is a fixed array inside the library.

Checked through the C ABI, on two calls in a row (the array keeps the
previous call's contents), against the fp64 oracle and against lr_linear
(the allocating entry point) on the same inputs, at the parity tolerance
used everywhere else; the device's free memory is the same before and after
the calls.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import lrgen
import oracle
from helpers import compare, to_dev, to_f64

pytestmark = pytest.mark.gpu

CASES = [
    (16, 256, 107, 256, False),      # the single-layer workload
    (1, 4096, 2867, 14336, False),   # decode gate/up, one token
    (4, 14336, 2867, 4096, True),    # decode down, four tokens, bias
    (16, 333, 257, 517, True),       # odd sizes everywhere
    (9, 64, 5, 9, True),
]


def _call_static(L, X, A, B, bias, Y, M, K, r, N, stream):
    return L.lr_linear_decode_static(X.data_ptr(), A.data_ptr(), B.data_ptr(),
                                     None if bias is None else bias.data_ptr(), Y.data_ptr(),
                                     M, K, r, N, stream)


@pytest.mark.parametrize("M,K,r,N,with_bias", CASES)
def test_static_matches_allocating_entry_point(M, K, r, N, with_bias):
    import torch
    import rank_linear_layers_b200 as lr
    L = lr.lib()
    stream = torch.cuda.current_stream().cuda_stream
    p = lrgen.lowrank_problem(M, K, r, N, seed=M * 7 + r, bias=with_bias)
    X, A, B, b = to_dev(p["X"]), to_dev(p["A"]), to_dev(p["B"]), to_dev(p["bias"])
    Yref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert L.lr_linear(X.data_ptr(), A.data_ptr(), B.data_ptr(),
                       None if b is None else b.data_ptr(), Yref.data_ptr(), M, K, r, N,
                       stream) == lr.LR_OK
    ref = to_f64(Yref)
    Yo = oracle.lr_linear(p["X"], p["A"], p["B"], p["bias"])
    Ys = [torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    # The first call on a device looks up the array's address; after it the
    # calls allocate nothing: free device memory is unchanged.
    assert _call_static(L, X, A, B, b, Ys[0], M, K, r, N, stream) == lr.LR_OK
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for call in range(2):
        Y = Ys[call]
        Y.fill_(float("nan"))
        assert _call_static(L, X, A, B, b, Y, M, K, r, N, stream) == lr.LR_OK
        torch.cuda.synchronize()
        compare(to_f64(Y), Yo, f"static call {call} vs oracle M={M} K={K} r={r} N={N}")
        compare(to_f64(Y), ref, f"static call {call} vs lr_linear M={M} K={K} r={r} N={N}")
    assert torch.cuda.mem_get_info()[0] == free0
    assert lr.last_device_status() == lr.LR_OK


def test_static_rejects_sizes_beyond_its_array():
    import torch
    import rank_linear_layers_b200 as lr
    L = lr.lib()
    stream = torch.cuda.current_stream().cuda_stream
    t = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    p = t.data_ptr()
    for (M, K, r, N) in [(17, 8, 8, 8), (1, 8, 4097, 8), (1, 8, 8, 16385)]:
        assert L.lr_linear_decode_static(p, p, p, None, p + 1024, M, K, r, N, stream) \
            == lr.LR_ERR_UNSUPPORTED

"""The r-split on one GPU: the layer's inner dimension cut into the slices
rsplit_bounds gives for three ranks, each slice's fp32 partial product from
lr_linear_rsplit (outside a process group: no reduction, the library's
kernels only), the partials summed on the device as the all-reduce would,
bias added by the first slice only — against the fp64 oracle of the whole
layer at the parity bar.  The reduction over real ranks is covered on CPU
ranks in test_dist.py."""
import numpy as np
import pytest

import lrgen
import oracle
from helpers import compare, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,r,N", [(64, 512, 300, 384), (4, 1000, 333, 700)])
def test_rsplit_slices_sum_to_the_layer(M, K, r, N):
    import torch
    from rank_linear_layers_b200 import rsplit
    p = lrgen.lowrank_problem(M, K, r, N, seed=21, bias=True)
    X = to_dev(p["X"])
    total = None
    for i in range(3):
        r0, r1 = rsplit.rsplit_bounds(r, 3, i)
        A = to_dev(np.ascontiguousarray(p["A"][:, r0:r1]))
        B = to_dev(np.ascontiguousarray(p["B"][r0:r1, :]))
        Y = rsplit.lr_linear_rsplit(X, A, B, to_dev(p["bias"]) if i == 0 else None)
        assert Y.dtype == torch.float32 and tuple(Y.shape) == (M, N)
        total = Y.clone() if total is None else total + Y
    torch.cuda.synchronize()
    compare(total.double().cpu().numpy(), oracle.lr_linear(p["X"], p["A"], p["B"], p["bias"]),
            f"r-split over 3 slices M={M} K={K} r={r} N={N}")

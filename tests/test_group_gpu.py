"""lr_linear_group on a full factorised Llama-3-8B decoder layer: q, k, v
share X; gate and up share X and write the two halves of one packed
[M, 2·N_int] buffer; o and down have their own inputs.  Ranks are drawn from
35-85% of min(K, N) (seed 7) and left unaligned; the pruned variant has
N_int = 12203 (odd row strides for gate/up/down and the packed output).

At M = 1 each projection is compared with the fp64 oracle; at M = 4096
each must equal lr_linear called on its own, bit for bit (the whole-output
oracle comparison of the M = 4096 layer is in test_full_size_gpu.py).
"""
import numpy as np
import pytest

import lrgen
import oracle
from helpers import compare, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_int", [14336, 12203])
@pytest.mark.parametrize("M", [1, 4096])
def test_decoder_layer_group(M, n_int):
    import torch
    import rank_linear_layers_b200 as lr
    layer = lrgen.decoder_layer(M, seed=7, n_int=n_int)
    xs = {k: to_dev(v) for k, v in layer["inputs"].items()}
    P = layer["projs"]
    dev = {n: (to_dev(p["A"]), to_dev(p["B"])) for n, p in P.items()}
    Ys = {n: torch.zeros((M, P[n]["N"]), dtype=torch.bfloat16, device="cuda")
          for n in ("q", "k", "v", "o", "down")}
    packed = torch.zeros((M, 2 * n_int), dtype=torch.bfloat16, device="cuda")
    entries = []
    for n, p in P.items():
        A, B = dev[n]
        e = dict(X=xs[p["x"]], A=A, B=B, K=p["K"], r=p["r"], N=p["N"])
        if n in ("gate", "up"):
            e["Y_ptr"] = packed.data_ptr() + (0 if n == "gate" else n_int * 2)
            e["ld_y"] = 2 * n_int
        else:
            e["Y"] = Ys[n]
        entries.append(e)
    # Tiles whole (no K range split between SMs), so that the group and the
    # single calls form every sum in the same order.
    lr.set_split_k(False)
    try:
        lr.lr_linear_group(entries, M)
        torch.cuda.synchronize()
    finally:
        lr.set_split_k(True)
    assert lr.last_device_status() == lr.LR_OK
    outs = {n: to_f64(Ys[n]) for n in Ys}
    pk = to_f64(packed)
    outs["gate"], outs["up"] = pk[:, :n_int], pk[:, n_int:]
    for n, p in P.items():
        X = layer["inputs"][p["x"]]
        # The same projection through lr_linear alone: the same bits on the
        # prefill path (tiles whole in both: tiling differs, sums do not); on
        # the decode path fp32 atomics may add partial sums in another order,
        # so compare at the parity tolerance there.
        A, B = dev[n]
        if M > 16:
            lr.set_split_k(False)
            try:
                Y1 = to_f64(lr.lr_linear(xs[p["x"]], A, B))
                torch.cuda.synchronize()
            finally:
                lr.set_split_k(True)
            assert np.array_equal(Y1, outs[n]), f"group vs single differ for {n}"
        else:
            Yr = oracle.lr_linear(X, p["A"], p["B"], None)
            compare(outs[n], Yr, f"{n} (r={p['r']}) M={M} N_int={n_int}")
            Y1 = to_f64(lr.lr_linear(xs[p["x"]], A, B))
            torch.cuda.synchronize()
            compare(outs[n], Y1, f"group vs single {n}")


def _group_case(specs, M, seed, split=True):
    """specs: list of (x_name, K, r, N, bias).  Returns inputs, entries, outputs."""
    import torch
    import rank_linear_layers_b200 as lr
    xs, entries, outs, probs = {}, [], [], []
    for i, (xn, K, r, N, bias) in enumerate(specs):
        p = lrgen.lowrank_problem(M, K, r, N, seed=seed + i, bias=bias)
        if xn not in xs:
            xs[xn] = (p["X"], to_dev(p["X"]))
        p["X"] = xs[xn][0]
        Y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
        e = dict(X=xs[xn][1], A=to_dev(p["A"]), B=to_dev(p["B"]), K=K, r=r, N=N, Y=Y)
        if bias:
            e["bias"] = to_dev(p["bias"])
        entries.append(e)
        outs.append(Y)
        probs.append(p)
    lr.set_split_k(split)
    try:
        lr.lr_linear_group(entries, M)
        torch.cuda.synchronize()
    finally:
        lr.set_split_k(True)
    assert lr.last_device_status() == lr.LR_OK
    return entries, outs, probs


@pytest.mark.parametrize("M", [17, 300])
def test_group_sets_share_x(M):
    """Sets of projections sharing X (concatenated factors, one GEMM1 per set,
    one launch), odd ranks and K, a misaligned X, bias on some: every output
    equals the oracle (tiles split along K between SMs, the default) and,
    with every tile whole, bit for bit the projection run alone."""
    import rank_linear_layers_b200 as lr
    specs = [("x1", 136, 37, 100, False), ("x1", 136, 64, 64, False), ("x1", 136, 5, 517, True),
             ("x2", 333, 257, 40, True), ("x2", 333, 1, 8, False), ("x3", 64, 7, 9, False),
             ("x4", 256, 128, 256, False)]
    entries, outs, probs = _group_case(specs, M, seed=40)
    for e, Y, p in zip(entries, outs, probs):
        compare(to_f64(Y), oracle.lr_linear(p["X"], p["A"], p["B"], p.get("bias")),
                f"group K={p['K']} r={p['r']} N={p['N']}")
    entries, outs, probs = _group_case(specs, M, seed=40, split=False)
    lr.set_split_k(False)
    try:
        for e, Y, p in zip(entries, outs, probs):
            Y1 = lr.lr_linear(e["X"], e["A"], e["B"], e.get("bias"))
            assert np.array_equal(to_f64(Y1), to_f64(Y)), f"group vs single r={p['r']}"
    finally:
        lr.set_split_k(True)


def test_group_larger_than_one_launch():
    """More projections than one launch's tables hold: run one by one."""
    specs = [(f"x{i % 3}", 96, 9 + i, 40 + i, i % 2 == 0) for i in range(14)]
    entries, outs, probs = _group_case(specs, 64, seed=70)
    for Y, p in zip(outs, probs):
        compare(to_f64(Y), oracle.lr_linear(p["X"], p["A"], p["B"], p.get("bias")),
                f"group(14) r={p['r']}")

"""The streamed decode kernel (one persistent launch for both products of a
decode call, M <= 8; lr_set_path(6) for single calls, the default for
decode-size groups) against the fp64 oracle, element by element, at the
parity bar of tests/helpers.py.

Covers: every token tile (M = 1..8), ragged ranks and widths (column blocks
of at most 248 with a partial last block), misaligned rows (odd row strides:
every row's window starts at another offset inside its 16-byte granule), W
whose first and last granules reach outside the tensor (bounded loads),
more column blocks than there are CTAs, bias, fp32 output, strided views,
repeated calls (the workspace must be zero again after each), agreement
with the two-launch decode kernels, and whole groups in one launch.
"""
import numpy as np
import pytest

import lrgen
import oracle
from helpers import compare, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lr():
    import torch
    import rank_linear_layers_b200 as lr
    lr.set_path(lr.PATH_AUTO)
    yield lr
    lr.set_path(lr.PATH_AUTO)
    torch.cuda.synchronize()


def ref(p):
    return oracle.lr_linear(p["X"], p["A"], p["B"], p["bias"])


def run(lr, p, path=6, y_f32=False):
    import torch
    lr.set_path(path)
    try:
        X, A, B, b = to_dev(p["X"]), to_dev(p["A"]), to_dev(p["B"]), to_dev(p["bias"])
        n0 = lr.kernel_launch_count()
        if y_f32:
            Y = lr.lr_linear_f32(X, A, B, b)
        else:
            Y = lr.lr_linear(X, A, B, b)
        launches = lr.kernel_launch_count() - n0
        torch.cuda.synchronize()
        assert lr.last_device_status() == lr.LR_OK
        return (Y.double().cpu().numpy() if y_f32 else to_f64(Y)), launches
    finally:
        lr.set_path(0)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("K,r,N", [(333, 107, 517), (64, 1, 9), (1000, 257, 2049),
                                   (4096, 2867, 1024), (130, 600, 300)])
def test_stream_ragged(lr, M, K, r, N):
    p = lrgen.lowrank_problem(M, K, r, N, seed=M * 31 + r, bias=(K % 2 == 0))
    Y, launches = run(lr, p)
    compare(Y, ref(p), f"stream M={M} K={K} r={r} N={N}")
    assert launches == 1


@pytest.mark.parametrize("M", [1, 4])
def test_stream_fp32_output(lr, M):
    p = lrgen.lowrank_problem(M, 700, 333, 1500, seed=3, bias=True)
    Y, _ = run(lr, p, y_f32=True)
    compare(Y, ref(p), f"stream fp32 M={M}")


def test_stream_many_blocks(lr):
    """N = 150000: 605 column blocks of 248, four CTAs' worth each; the host
    checks every CTA's piece count."""
    p = lrgen.lowrank_problem(1, 256, 40, 150000, seed=4, bias=True)
    Y, _ = run(lr, p)
    compare(Y, ref(p), "stream N=150000")


def test_stream_edges_outside_tensor(lr):
    """A and B start 2 bytes past a 16-byte boundary and end 2 bytes before
    one, with odd row strides: the first granule of the first row and the
    last granule of the last row reach outside the tensors."""
    import torch
    M, K, r, N = 3, 77, 45, 333
    p = lrgen.lowrank_problem(M, K, r, N, seed=9, bias=True)

    def off(bits):
        t = to_dev(bits).reshape(-1)
        buf = torch.zeros(t.numel() + 16, dtype=torch.bfloat16, device="cuda")
        buf[1:1 + t.numel()] = t
        return buf[1:1 + t.numel()].view(bits.shape)

    X, A, B, b = off(p["X"]), off(p["A"]), off(p["B"]), off(p["bias"])
    assert A.data_ptr() % 16 == 2 and B.data_ptr() % 16 == 2
    lr.set_path(6)
    try:
        Y = lr.lr_linear(X, A, B, b)
    finally:
        lr.set_path(0)
    torch.cuda.synchronize()
    assert lr.last_device_status() == lr.LR_OK
    compare(to_f64(Y), ref(p), "stream edges")


@pytest.mark.parametrize("M", [1, 5])
def test_stream_strided_views(lr, M):
    """Operands as views of wider buffers with odd pitches."""
    import torch
    K, r, N = 500, 123, 999
    p = lrgen.lowrank_problem(M, K, r, N, seed=12, bias=False)

    def view(bits, pitch):
        t = to_dev(bits)
        buf = torch.zeros((t.shape[0], pitch), dtype=torch.bfloat16, device="cuda")
        buf[:, :t.shape[1]] = t
        return buf[:, :t.shape[1]]

    X, A, B = view(p["X"], K + 3), view(p["A"], r + 5), view(p["B"], N + 1)
    lr.set_path(6)
    try:
        Y = lr.lr_linear_strided(X, A, B)
    finally:
        lr.set_path(0)
    torch.cuda.synchronize()
    assert lr.last_device_status() == lr.LR_OK
    compare(to_f64(Y), ref(p), f"stream strided M={M}")


def test_stream_repeated_and_interleaved(lr):
    """Calls of different shapes, on the streamed and the two-launch
    kernels in turn, share the zero-at-rest workspace."""
    cases = [lrgen.lowrank_problem(4, 1024, 300, 2000, seed=5),
             lrgen.lowrank_problem(16, 700, 1000, 129, seed=6, bias=True),
             lrgen.lowrank_problem(1, 4096, 2867, 4096, seed=7),
             lrgen.lowrank_problem(8, 257, 31, 4100, seed=8, bias=True)]
    refs = [ref(p) for p in cases]
    for _ in range(3):
        for p, Yr in zip(cases, refs):
            compare(run(lr, p)[0], Yr, "stream repeated")
            compare(run(lr, p, path=5)[0], Yr, "two-launch repeated")


@pytest.mark.parametrize("M", [1, 4])
@pytest.mark.parametrize("proj", ["gate_up", "down"])
def test_stream_matches_two_launch_kernels(lr, M, proj):
    """The decode MLP shapes on both decode kernels: each within the bar of
    the oracle and of each other."""
    K, N = (4096, 14336) if proj == "gate_up" else (14336, 4096)
    p = lrgen.lowrank_problem(M, K, 2867, N, seed=0)
    Ys, launches = run(lr, p, path=6)
    Yt, _ = run(lr, p, path=5)
    Yr = ref(p)
    compare(Ys, Yr, f"stream {proj} M={M}")
    compare(Yt, Yr, f"two-launch {proj} M={M}")
    compare(Ys, Yt, f"stream vs two-launch {proj} M={M}")
    assert launches == 1


@pytest.mark.parametrize("M", [1, 3, 8])
def test_group_in_one_launch(lr, M):
    """A decode-size group (odd ranks, shared and separate X, bias on some,
    an fp32 output, a packed output with row stride 2·N) is one launch; every
    output equals the oracle."""
    import torch
    specs = [("x1", 4096, 1475, 4096, False), ("x1", 4096, 553, 1024, True),
             ("x1", 4096, 826, 1024, False), ("x2", 4096, 2315, 4096, True),
             ("x3", 4096, 1505, 2000, False), ("x3", 4096, 2125, 2000, False),
             ("x4", 14336, 1691, 4096, True)]
    xs, entries, probs, outs = {}, [], [], []
    packed = torch.zeros((M, 4000), dtype=torch.bfloat16, device="cuda")
    for i, (xn, K, r, N, bias) in enumerate(specs):
        p = lrgen.lowrank_problem(M, K, r, N, seed=90 + i, bias=bias)
        if xn not in xs:
            xs[xn] = (p["X"], to_dev(p["X"]))
        p["X"] = xs[xn][0]
        e = dict(X=xs[xn][1], A=to_dev(p["A"]), B=to_dev(p["B"]), K=K, r=r, N=N)
        if bias:
            e["bias"] = to_dev(p["bias"])
        if i in (4, 5):
            e["Y_ptr"] = packed.data_ptr() + (0 if i == 4 else 2000 * 2)
            e["ld_y"] = 4000
            outs.append(("packed", i))
        else:
            dt = torch.float32 if i == 2 else torch.bfloat16
            e["Y"] = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
            outs.append(("own", i))
        entries.append(e)
        probs.append(p)
    n0 = lr.kernel_launch_count()
    lr.lr_linear_group(entries, M)
    launches = lr.kernel_launch_count() - n0
    torch.cuda.synchronize()
    assert lr.last_device_status() == lr.LR_OK
    assert launches == 1
    pk = to_f64(packed)
    for (kind, i), e, p in zip(outs, entries, probs):
        if kind == "packed":
            Y = pk[:, :2000] if i == 4 else pk[:, 2000:]
        elif e["Y"].dtype == torch.float32:
            Y = e["Y"].double().cpu().numpy()
        else:
            Y = to_f64(e["Y"])
        compare(Y, ref(p), f"group M={M} projection {i}")

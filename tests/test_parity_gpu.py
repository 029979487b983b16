"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bar (bf16 inputs, fp32 accumulation): max|err| <= 2e-2·RMS(Y_ref) and
relative Frobenius error <= 5e-3, on every output (tests/helpers.py), with
no other allowance.  These cases compare every element; the full-size
workloads are in test_full_size_gpu.py.
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
    yield lr
    lr.set_path(lr.PATH_AUTO)
    torch.cuda.synchronize()


def run_gpu(lr, p, path=0, bias=None):
    import torch
    lr.set_path(path)
    try:
        X, A, B = to_dev(p["X"]), to_dev(p["A"]), to_dev(p["B"])
        b = to_dev(p["bias"] if bias is None else bias)
        Y = lr.lr_linear(X, A, B, b)
        torch.cuda.synchronize()
        assert lr.last_device_status() == lr.LR_OK
        return to_f64(Y)
    finally:
        lr.set_path(0)


def ref(p, rows=None):
    return oracle.lr_linear(p["X"], p["A"], p["B"], p["bias"], rows=rows)


# ---------------------------------------------------------------- decode
def test_single_layer_m16_k256_r107(lr):
    # X [16,256] ~N(0,1), A [256,107], B [107,256] ~N(0,1/fan_in), no bias, seed 0.
    p = lrgen.lowrank_problem(16, 256, 107, 256, seed=0)
    Yr = ref(p)
    compare(run_gpu(lr, p), Yr, "c1 auto")
    compare(run_gpu(lr, p, lr.PATH_DECODE), Yr, "c1 decode")
    compare(run_gpu(lr, p, lr.PATH_PREFILL), Yr, "c1 prefill")


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 16])
@pytest.mark.parametrize("r", [1, 7, 8, 9, 63, 65, 107, 255, 257, 300])
def test_decode_ragged(lr, M, r):
    K, N = 333, 517
    p = lrgen.lowrank_problem(M, K, r, N, seed=1000 + r, bias=(r % 2 == 1))
    compare(run_gpu(lr, p, lr.PATH_DECODE), ref(p), f"decode M={M} r={r}")


@pytest.mark.parametrize("K,N", [(8, 8), (1, 1000), (4096, 40), (130, 2049)])
def test_decode_shapes(lr, K, N):
    p = lrgen.lowrank_problem(4, K, 37, N, seed=7, bias=True)
    compare(run_gpu(lr, p, lr.PATH_DECODE), ref(p), f"decode K={K} N={N}")
    p = lrgen.lowrank_problem(16, K, 37, N, seed=8, bias=True)
    compare(run_gpu(lr, p, lr.PATH_DECODE), ref(p), f"decode16 K={K} N={N}")


@pytest.mark.parametrize("M,K,r,N", [(1, 333, 57, 77), (5, 256, 107, 256), (16, 200, 33, 517),
                                     (16, 1000, 9, 130), (3, 64, 1, 8)])
def test_tiny_layer_one_cta(lr, M, K, r, N):
    """Small layers (automatic dispatch): the whole layer in one CTA, odd
    sizes and bias, bf16 and fp32 outputs, operands not 16-byte aligned."""
    import torch
    p = lrgen.lowrank_problem(M, K, r, N, seed=M * 7 + r, bias=True)
    Yr = ref(p)
    n0 = lr.kernel_launch_count()
    compare(run_gpu(lr, p), Yr, f"tiny {M}x{K}x{r}x{N}")
    assert lr.kernel_launch_count() - n0 == 1

    def off(bits):
        t = to_dev(bits).reshape(-1)
        buf = torch.empty(t.numel() + 1, dtype=torch.bfloat16, device="cuda")
        buf[1:] = t
        return buf[1:].view(bits.shape)
    Y32 = lr.lr_linear_f32(off(p["X"]), off(p["A"]), off(p["B"]), off(p["bias"]))
    torch.cuda.synchronize()
    compare(f32_host(Y32), Yr, "tiny fp32, unaligned operands")


# ---------------------------------------------------------------- prefill
@pytest.mark.parametrize("M,K,r,N", [
    (128, 64, 64, 256),       # one tile each way, all aligned
    (128, 128, 256, 256),
    (200, 256, 107, 300),     # odd r (A rows 2-byte aligned), ragged M and N
    (300, 333, 257, 517),     # odd K too (X rows misaligned)
    (17, 64, 1, 8),           # smallest prefill M, rank 1
    (129, 1000, 511, 1000),
    (256, 512, 1741 // 4, 700),
    (384, 4096, 1741, 256),   # full-depth K, c2's rank
])
def test_prefill_ragged(lr, M, K, r, N):
    p = lrgen.lowrank_problem(M, K, r, N, seed=M + K + r + N, bias=True)
    compare(run_gpu(lr, p, lr.PATH_PREFILL), ref(p), f"prefill {M}x{K}x{r}x{N}")


@pytest.mark.parametrize("M,K,r,N", [
    (256, 512, 256, 512),      # one pair tile
    (300, 333, 257, 517),      # ragged everywhere, odd K and r
    (640, 1024, 1741, 700),
])
def test_pair_and_single_sm_kernels_agree(lr, M, K, r, N):
    p = lrgen.lowrank_problem(M, K, r, N, seed=M + r, bias=True)
    Yp = run_gpu(lr, p, lr.PATH_PREFILL_PAIR)
    Y1 = run_gpu(lr, p, lr.PATH_PREFILL_1SM)
    Yr = ref(p)
    compare(Yp, Yr, "pair kernel")
    compare(Y1, Yr, "single-SM kernel")


@pytest.mark.parametrize("t_mode", [1, 2])
@pytest.mark.parametrize("bn", [32, 64, 96, 128, 160, 192, 224, 256])
def test_prefill_forced_tile_width(lr, bn, t_mode):
    """Every tile width the planner may pick, on a ragged shape (odd K, r, N;
    partial 64-column atoms when bn is not a multiple of 64; Y rows not
    16-byte aligned, so Y takes the per-thread stores and T the TMA stores),
    with T rounded once (every width) and in two parts (GEMM2 capped at 128
    columns, where both parts of T share a stage with the b tile)."""
    p = lrgen.lowrank_problem(300, 333, 257, 517, seed=bn, bias=True)
    lr.set_tile_n(bn)
    lr.set_t_precision(t_mode)
    try:
        Y = run_gpu(lr, p, lr.PATH_PREFILL)
    finally:
        lr.set_tile_n(0)
        lr.set_t_precision(lr.T_AUTO)
    compare(Y, ref(p), f"prefill bn={bn} t_mode={t_mode}")


@pytest.mark.parametrize("M,K,r,N", [
    (300, 2048, 37, 300),     # 3 GEMM1 tiles, 32 k blocks: split 4 ways
    (129, 1000, 8, 77),       # ragged M, K not a multiple of 64
    (640, 4096, 64, 1000),
])
def test_prefill_split_k(lr, M, K, r, N):
    """GEMM1 with too few tiles splits its K loop over CTAs (fp32 partial
    sums, the last split rounds T); the same with splitting turned off."""
    p = lrgen.lowrank_problem(M, K, r, N, seed=K + r, bias=True)
    Ys = run_gpu(lr, p, lr.PATH_PREFILL)
    lr.set_split_k(False)
    try:
        Y1 = run_gpu(lr, p, lr.PATH_PREFILL)
    finally:
        lr.set_split_k(True)
    Yr = ref(p)
    compare(Ys, Yr, f"split-K {M}x{K}x{r}x{N}")
    compare(Y1, Yr, f"no split {M}x{K}x{r}x{N}")
    # Repeated calls: the split workspace must be zero again after each (a
    # left-over partial sum would double-count).  The fp32 reductions add the
    # splits in a run-dependent order, so the bits may differ.
    for _ in range(2):
        compare(run_gpu(lr, p, lr.PATH_PREFILL), Yr, "split-K repeated")


def test_dense_split_k(lr):
    """lr_dense with a long K and few tiles (split K), bias, ragged N."""
    import torch
    M, K, N = 256, 8192, 70
    p = lrgen.lowrank_problem(M, K, N, 1, seed=5, bias=False)
    bias = lrgen.lowrank_problem(1, 1, 1, N, seed=6, bias=True)["bias"]
    X, W = to_dev(p["X"]), to_dev(p["A"])
    Y = lr.lr_dense(X, W, to_dev(bias))
    torch.cuda.synchronize()
    eye = np.zeros((N, N), dtype=np.uint16)
    eye[np.arange(N), np.arange(N)] = 0x3F80  # bf16 1.0: X·W·I through the oracle
    compare(to_f64(Y), oracle.lr_linear(p["X"], p["A"], eye, bias), "dense split-K")


def test_decode_and_prefill_agree_at_m16(lr):
    p = lrgen.lowrank_problem(16, 512, 300, 640, seed=3, bias=True)
    Yd = run_gpu(lr, p, lr.PATH_DECODE)
    Yp = run_gpu(lr, p, lr.PATH_PREFILL)
    Yr = ref(p)
    compare(Yd, Yr, "decode")
    compare(Yp, Yr, "prefill")
    compare(Yd, Yp, "decode vs prefill")


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("M,K,r,N", [
    (300, 333, 257, 517),     # odd K, r and N, bias
    (640, 4096, 64, 1000),    # GEMM1 splits K
    (200, 256, 107, 300),
])
def test_prefill_t_precision_modes(lr, mode, M, K, r, N):
    """T rounded once (1) and T in two parts (2), each forced: fp32 and bf16
    outputs against the oracle."""
    import torch
    p = lrgen.lowrank_problem(M, K, r, N, seed=3 * M + r, bias=True)
    X, A, B, b = to_dev(p["X"]), to_dev(p["A"]), to_dev(p["B"]), to_dev(p["bias"])
    Yr = ref(p)
    lr.set_t_precision(mode)
    try:
        Y32 = lr.lr_linear_f32(X, A, B, b)
        Y16 = lr.lr_linear(X, A, B, b)
        torch.cuda.synchronize()
    finally:
        lr.set_t_precision(lr.T_AUTO)
    assert lr.last_device_status() == lr.LR_OK
    compare(f32_host(Y32), Yr, f"mode {mode} fp32")
    compare(to_f64(Y16), Yr, f"mode {mode} bf16")


@pytest.mark.parametrize("path", [1, 2])
@pytest.mark.parametrize("M,K,r,N", [(4, 333, 257, 517), (16, 512, 300, 640), (129, 1000, 511, 1000)])
def test_fp32_output(lr, path, M, K, r, N):
    """lr_linear_f32 on the decode path (M <= 16) and the prefill path: the
    accumulator plus bias, unrounded, against the oracle; also an empty
    contraction (Y = bias in fp32)."""
    import torch
    if path == 1 and M > 16:
        pytest.skip("decode path takes M <= 16")
    p = lrgen.lowrank_problem(M, K, r, N, seed=M + r + path, bias=True)
    lr.set_path(path)
    try:
        Y32 = lr.lr_linear_f32(to_dev(p["X"]), to_dev(p["A"]), to_dev(p["B"]), to_dev(p["bias"]))
        torch.cuda.synchronize()
    finally:
        lr.set_path(0)
    assert lr.last_device_status() == lr.LR_OK
    compare(f32_host(Y32), ref(p), f"fp32 path={path}")
    Z = lr.lr_linear_f32(torch.zeros((M, K), dtype=torch.bfloat16, device="cuda"),
                         torch.zeros((K, 0), dtype=torch.bfloat16, device="cuda"),
                         torch.zeros((0, N), dtype=torch.bfloat16, device="cuda"), to_dev(p["bias"]))
    torch.cuda.synchronize()
    assert np.array_equal(f32_host(Z), np.broadcast_to(lrgen.bf16_to_f64(p["bias"]), (M, N)))


@pytest.mark.parametrize("M,K,r,N", [(300, 333, 257, 517), (2048, 1024, 1741, 4096), (4, 4096, 333, 700)])
def test_strided_operands_and_prepared_factors(lr, M, K, r, N):
    """lr_linear_strided with padded row pitches for X, A, B and Y (bf16 and
    fp32 outputs) against the oracle; with every prefill operand 32-byte
    aligned at a 16-element pitch (factors in lr_factor_pitch buffers) the
    call is one launch: no realignment copy."""
    import torch
    p = lrgen.lowrank_problem(M, K, r, N, seed=K + r, bias=True)
    Yr = ref(p)

    def padded(bits, pitch):
        rows, cols = bits.shape
        buf = torch.zeros((rows, pitch), dtype=torch.bfloat16, device="cuda")
        buf[:, :cols] = to_dev(bits)
        return buf[:, :cols]
    X = padded(p["X"], lr.factor_pitch(K))
    A = padded(p["A"], lr.factor_pitch(r))
    B = padded(p["B"], lr.factor_pitch(N))
    b = to_dev(p["bias"])
    assert A.stride(0) == lr.factor_pitch(r) and lr.factor_pitch(r) % 64 == 0
    Ybuf = torch.zeros((M, N + 3), dtype=torch.bfloat16, device="cuda")
    n0 = lr.kernel_launch_count()
    lr.lr_linear_strided(X, A, B, b, Y=Ybuf[:, :N])
    torch.cuda.synchronize()
    if M > 16:
        assert lr.kernel_launch_count() - n0 == 1, "prepared operands must not be copied"
    assert lr.last_device_status() == lr.LR_OK
    compare(to_f64(Ybuf[:, :N].contiguous()), Yr, f"strided bf16 {M}x{K}x{r}x{N}")
    assert np.all(to_f64(Ybuf[:, N:].contiguous()) == 0.0), "wrote past N"
    Y32 = torch.zeros((M, N + 1), dtype=torch.float32, device="cuda")
    lr.lr_linear_strided(X, A, B, b, Y=Y32[:, :N])
    torch.cuda.synchronize()
    compare(f32_host(Y32[:, :N]), Yr, f"strided fp32 {M}x{K}x{r}x{N}")


# ---------------------------------------------------------------- edges
def test_empty_and_degenerate(lr):
    import torch
    # r = 0 and K = 0: Y = bias.
    for (M, K, r, N) in [(5, 8, 0, 9), (40, 0, 3, 9), (3, 0, 0, 4)]:
        p = lrgen.lowrank_problem(M, K, r, N, seed=1, bias=True)
        X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
        A = torch.zeros((K, r), dtype=torch.bfloat16, device="cuda")
        B = torch.zeros((r, N), dtype=torch.bfloat16, device="cuda")
        b = to_dev(p["bias"])
        Y = lr.lr_linear(X, A, B, b)
        assert np.array_equal(to_f64(Y), np.broadcast_to(lrgen.bf16_to_f64(p["bias"]), (M, N)))
    # M = 0 or N = 0: nothing to do.
    X = torch.zeros((0, 8), dtype=torch.bfloat16, device="cuda")
    Y = lr.lr_linear(X, torch.zeros((8, 3), dtype=torch.bfloat16, device="cuda"),
                     torch.zeros((3, 5), dtype=torch.bfloat16, device="cuda"))
    assert Y.shape == (0, 5)


def test_unaligned_base_pointers(lr):
    """Views that start 2 bytes into a buffer: no operand is 16-byte aligned."""
    import torch
    for (M, K, r, N, path) in [(200, 136, 64, 264, 2), (8, 136, 64, 264, 1)]:
        p = lrgen.lowrank_problem(M, K, r, N, seed=21, bias=True)
        def off(bits):
            t = to_dev(bits).reshape(-1)
            buf = torch.empty(t.numel() + 1, dtype=torch.bfloat16, device="cuda")
            buf[1:] = t
            return buf[1:].view(bits.shape)
        X, A, B, b = off(p["X"]), off(p["A"]), off(p["B"]), off(p["bias"])
        ybuf = torch.empty(M * N + 1, dtype=torch.bfloat16, device="cuda")
        Y = ybuf[1:].view(M, N)
        assert X.data_ptr() % 16 != 0 and Y.data_ptr() % 16 != 0
        lr.set_path(path)
        try:
            lr.lr_linear(X, A, B, b, Y=Y)
        finally:
            lr.set_path(0)
        torch.cuda.synchronize()
        compare(to_f64(Y), ref(p), f"unaligned path={path}")


def test_repeated_calls_reuse_workspace(lr):
    """The decode workspace must be zero again after each call (self-cleaning)."""
    p = lrgen.lowrank_problem(4, 1024, 300, 2000, seed=5)
    q = lrgen.lowrank_problem(16, 700, 1000, 129, seed=6, bias=True)
    Yp, Yq = ref(p), ref(q)
    for _ in range(3):
        compare(run_gpu(lr, p, lr.PATH_DECODE), Yp, "p")
        compare(run_gpu(lr, q, lr.PATH_DECODE), Yq, "q")


# ---------------------------------------------------------------- full size
@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("proj", ["gate_up", "down"])
def test_decode_mlp_full_size(lr, M, proj):
    K, N = (4096, 14336) if proj == "gate_up" else (14336, 4096)
    p = lrgen.lowrank_problem(M, K, 2867, N, seed=0)
    compare(run_gpu(lr, p), ref(p), f"decode {proj} M={M}")

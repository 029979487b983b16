"""Whole-output parity at the full workload sizes, against the fp64 oracle.

Every element of every output is compared (no sampling):
  * the prefill q_proj workload, M=2048, K=N=4096, r=1741, A = U·Σ, B = Vᵀ;
  * the misalignment sweep, M=K=N=4096, at r = 64, 128, 512, 1000, 1004,
    1024, 1025, 1032, 1089, 1100 and 2048;
  * a full factorised Llama-3-8B decoder layer through lr_linear_group at
    M=4096, both N_int = 14336 and the pruned N_int = 12203.

The bar (max|err| <= 2e-2·RMS, relative Frobenius <= 5e-3) is stated for
bf16 inputs with fp32 accumulation and is checked on the library's fp32
output.  The bf16 output adds one rounding of up to 2^-8·|Y|: at the q_proj
workload the exact result rounded once to bf16 already misses the bar
(2.18e-2·RMS at its largest output, 6.7·RMS), so no bf16 result can meet it
there.  The bf16 output is therefore checked to be exactly the fp32 output
rounded to nearest-even (split K off, so both calls add their sums in one
order), and, where T is carried in two parts (its bf16 rounding removed),
against the oracle at the same bar.
"""
import numpy as np
import pytest

import lrgen
import oracle
from helpers import compare, f32_host, rn_bf16, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lr():
    import torch
    import rank_linear_layers_b200 as lr
    lr.set_path(lr.PATH_AUTO)
    lr.set_t_precision(lr.T_AUTO)
    yield lr
    lr.set_split_k(True)
    lr.set_t_precision(lr.T_AUTO)
    torch.cuda.synchronize()


def _run(lr, fn, *args):
    import torch
    Y = fn(*args)
    torch.cuda.synchronize()
    assert lr.last_device_status() == lr.LR_OK
    return Y


def check_all_forms(lr, p, what, two_part_bf16_meets_bar=True):
    """fp32 output vs the oracle; bf16 output == RN(fp32 output); bf16 output
    with T in two parts vs the oracle."""
    X, A, B = to_dev(p["X"]), to_dev(p["A"]), to_dev(p["B"])
    bias = to_dev(p["bias"]) if p.get("bias") is not None else None
    Yr = oracle.lr_linear(p["X"], p["A"], p["B"], p.get("bias"))
    Y32 = _run(lr, lr.lr_linear_f32, X, A, B, bias)
    compare(f32_host(Y32), Yr, f"{what} fp32 output")
    lr.set_split_k(False)
    try:
        Y32s = _run(lr, lr.lr_linear_f32, X, A, B, bias)
        Y16s = _run(lr, lr.lr_linear, X, A, B, bias)
    finally:
        lr.set_split_k(True)
    assert np.array_equal(to_f64(Y16s), rn_bf16(Y32s)), \
        f"{what}: bf16 output is not the fp32 output rounded to nearest-even"
    lr.set_t_precision(lr.T_TWO_PARTS)
    try:
        Y16t = _run(lr, lr.lr_linear, X, A, B, bias)
        Y32t = _run(lr, lr.lr_linear_f32, X, A, B, bias)
    finally:
        lr.set_t_precision(lr.T_AUTO)
    compare(f32_host(Y32t), Yr, f"{what} fp32 output, T in two parts")
    if two_part_bf16_meets_bar:
        compare(to_f64(Y16t), Yr, f"{what} bf16 output, T in two parts")
    return Yr


def test_q_proj_whole_output(lr):
    p = lrgen.svd_problem(M=2048, K=4096, N=4096, r=1741, seed=0)
    Yr = check_all_forms(lr, p, "q_proj", two_part_bf16_meets_bar=False)
    # The documented reason the bf16 form is exempt: the exact result rounded
    # once to bf16 misses the bar at this workload.
    rms = float(np.sqrt(np.mean(Yr ** 2)))
    exact_rn = float(np.abs(rn_bf16(Yr.astype(np.float32)) - Yr).max()) / rms
    assert exact_rn > 2e-2, exact_rn


@pytest.mark.parametrize("r", [64, 128, 512, 1000, 1004, 1024, 1025, 1032, 1089, 1100, 2048])
def test_sweep_whole_output(lr, r):
    p = lrgen.lowrank_problem(4096, 4096, r, 4096, seed=r)
    check_all_forms(lr, p, f"M=K=N=4096 r={r}")


@pytest.mark.parametrize("n_int", [14336, 12203])
def test_decoder_layer_whole_outputs(lr, n_int):
    """lr_linear_group at M=4096: the fp32 outputs of every projection against
    the oracle, and the bf16 outputs equal to them rounded to nearest-even."""
    import torch
    M = 4096
    layer = lrgen.decoder_layer(M, seed=7, n_int=n_int)
    xs = {k: to_dev(v) for k, v in layer["inputs"].items()}
    P = layer["projs"]
    dev = {n: (to_dev(p["A"]), to_dev(p["B"])) for n, p in P.items()}

    def run(dtype):
        outs = {n: torch.zeros((M, P[n]["N"]), dtype=dtype, device="cuda")
                for n in ("q", "k", "v", "o", "down")}
        packed = torch.zeros((M, 2 * n_int), dtype=dtype, device="cuda")
        es = packed.element_size()
        entries = []
        for n, p in P.items():
            A, B = dev[n]
            e = dict(X=xs[p["x"]], A=A, B=B, K=p["K"], r=p["r"], N=p["N"],
                     y_f32=dtype == torch.float32)
            if n in ("gate", "up"):
                e["Y_ptr"] = packed.data_ptr() + (0 if n == "gate" else n_int * es)
                e["ld_y"] = 2 * n_int
            else:
                e["Y"] = outs[n]
            entries.append(e)
        _run(lr, lr.lr_linear_group, entries, M)
        outs["gate"], outs["up"] = packed[:, :n_int], packed[:, n_int:]
        return outs

    lr.set_split_k(False)
    try:
        y32 = run(torch.float32)
        y16 = run(torch.bfloat16)
    finally:
        lr.set_split_k(True)
    for n, p in P.items():
        Yr = oracle.lr_linear(layer["inputs"][p["x"]], p["A"], p["B"], None)
        compare(f32_host(y32[n]), Yr, f"{n} (K={p['K']} r={p['r']} N={p['N']}) fp32 output")
        assert np.array_equal(to_f64(y16[n].contiguous()), rn_bf16(y32[n])), \
            f"{n}: bf16 output is not the fp32 output rounded to nearest-even"

"""Shared helpers for the GPU parity tests: move generator bits to the GPU,
read results back, and compare with the oracle at the stated tolerance.

Tolerance (bf16 inputs, fp32 accumulation), on every compared output:
    max |Y_gpu - Y_ref| <= 2e-2 · RMS(Y_ref)
    ||Y_gpu - Y_ref||_F / ||Y_ref||_F <= 5e-3
Y_gpu is the library's fp32 output (lr_linear_f32) or its bf16 output.  A
bf16 output carries one more rounding, up to 2^-8·|Y| per element; where
even the exact result rounded once to bf16 breaks the bar (the prefill
q_proj workload: its largest output is 6.7·RMS), the tests check the fp32
output against the oracle and the bf16 output for equality with that fp32
output rounded to nearest-even.
"""
import numpy as np

import lrgen

MAX_ERR_RMS = 2e-2
REL_FRO = 5e-3


def to_dev(bits, device="cuda"):
    import torch
    if bits is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def to_f64(t):
    import torch
    return lrgen.bf16_to_f64(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def compare(Y, Yref, what=""):
    """Assert the parity bar; returns (max_err/rms, rel_fro)."""
    Y = np.asarray(Y, dtype=np.float64)
    Yref = np.asarray(Yref, dtype=np.float64)
    assert Y.shape == Yref.shape, (what, Y.shape, Yref.shape)
    assert np.all(np.isfinite(Y)), f"{what}: non-finite output"
    rms = float(np.sqrt(np.mean(Yref ** 2))) if Yref.size else 0.0
    err = np.abs(Y - Yref)
    if rms == 0.0:
        assert np.all(err == 0.0), f"{what}: expected exact zeros/bias"
        return 0.0, 0.0
    mx = float(err.max()) / rms
    rel = float(np.linalg.norm(Y - Yref) / np.linalg.norm(Yref))
    assert mx <= MAX_ERR_RMS, f"{what}: max|err| = {mx:.3e}·RMS > {MAX_ERR_RMS}"
    assert rel <= REL_FRO, f"{what}: rel Frobenius {rel:.3e} > {REL_FRO}"
    return mx, rel


def rn_bf16(Y32):
    """fp32 values (numpy or torch) rounded to nearest-even bf16, as float64
    (torch's conversion): what the library's bf16 output must equal when it
    is the same fp32 accumulator rounded once."""
    import torch
    t = Y32 if isinstance(Y32, torch.Tensor) else torch.from_numpy(np.asarray(Y32, np.float32))
    return t.detach().cpu().float().to(torch.bfloat16).double().numpy()


def f32_host(Y32):
    """A device fp32 tensor as float64 numpy (exact)."""
    return Y32.detach().cpu().double().numpy()

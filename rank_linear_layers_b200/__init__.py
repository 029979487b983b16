"""rank_linear_layers_b200 — B200 (sm_100a) low-rank linear layer Y = (X·A)·B (+bias).

A thin ctypes binding over ``liblrlinear.so`` (C ABI in ``include/lr_linear.h``).
This module only marshals arguments: torch tensors supply device pointers and
the current CUDA stream; every step of the layer runs in the library's CUDA
kernels.  There is no CPU or PyTorch fallback: if the library is missing or
was built for another GPU, calls raise.

    import torch, rank_linear_layers_b200 as lr
    Y = lr.lr_linear(X, A, B)            # X [M,K], A [K,r], B [r,N] bf16 cuda
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblrlinear.so")

LR_OK = 0
LR_ERR_INVALID_ARG = 1
LR_ERR_UNSUPPORTED = 2
LR_ERR_CUDA = 3
LR_ERR_TIMEOUT = 4
LR_ERR_NO_MEMORY = 5
LR_ERR_INFEASIBLE = 6

PATH_AUTO, PATH_DECODE, PATH_PREFILL, PATH_PREFILL_1SM, PATH_PREFILL_PAIR = 0, 1, 2, 3, 4
PATH_DECODE_TWO_LAUNCH, PATH_DECODE_STREAM = 5, 6

# Every symbol include/lr_linear.h declares.
EXPORTS = (
    "lr_linear", "lr_linear_f32", "lr_linear_group", "lr_linear_host", "lr_dense",
    "lr_last_device_status",
    "lr_status_string", "lr_last_cuda_error", "lr_set_path", "lr_set_wait_limit_ns",
    "lr_kernel_launch_count", "lr_release_workspaces", "lr_linear_decode_static",
    "lr_set_withhold_first_stage", "lr_set_tile_n", "lr_set_split_k", "lr_set_early_copy",
    "lr_gac_select", "lr_set_t_precision", "lr_linear_strided", "lr_factor_pitch",
)

T_AUTO, T_BF16, T_TWO_PARTS = 0, 1, 2


class LrError(RuntimeError):
    def __init__(self, code: int, what: str, cuda_error: int = 0):
        self.code = code
        self.cuda_error = cuda_error
        super().__init__(f"{what}: {status_string(code)} (cuda error {cuda_error})")


class LrProj(ctypes.Structure):
    _fields_ = [
        ("X", ctypes.c_void_p), ("K", ctypes.c_int64), ("A", ctypes.c_void_p),
        ("B", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("Y", ctypes.c_void_p),
        ("ld_y", ctypes.c_int64), ("r", ctypes.c_int64), ("N", ctypes.c_int64),
        ("y_f32", ctypes.c_int32), ("silu_gate", ctypes.c_int32),
    ]


_lib = None


def lib(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m rank_linear_layers_b200.build` "
            "(there is no fallback implementation)")
    L = ctypes.CDLL(path)
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    L.lr_linear.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
    L.lr_linear_f32.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
    L.lr_linear_strided.argtypes = [vp, i64, vp, i64, vp, i64, vp, vp, i64, i64, i64, i64, i64,
                                    ctypes.c_int32, vp]
    L.lr_factor_pitch.argtypes = [i64]
    L.lr_factor_pitch.restype = i64
    L.lr_linear_group.argtypes = [ctypes.POINTER(LrProj), ctypes.c_int, i64, vp]
    L.lr_linear_host.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
    L.lr_dense.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp]
    L.lr_linear_decode_static.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
    L.lr_last_device_status.argtypes = [vp]
    L.lr_status_string.argtypes = [ctypes.c_int]
    L.lr_status_string.restype = ctypes.c_char_p
    L.lr_last_cuda_error.argtypes = []
    L.lr_set_path.argtypes = [ctypes.c_int]
    L.lr_set_wait_limit_ns.argtypes = [i64]
    L.lr_set_withhold_first_stage.argtypes = [ctypes.c_int]
    L.lr_set_tile_n.argtypes = [ctypes.c_int]
    L.lr_set_split_k.argtypes = [ctypes.c_int]
    L.lr_set_early_copy.argtypes = [ctypes.c_int]
    L.lr_set_t_precision.argtypes = [ctypes.c_int]
    ip, lp, dp = (ctypes.POINTER(ctypes.c_int), ctypes.POINTER(i64),
                  ctypes.POINTER(ctypes.c_double))
    L.lr_gac_select.argtypes = [ctypes.c_int, ip, lp, dp, lp, i64, i64, ip, dp]
    L.lr_kernel_launch_count.argtypes = []
    L.lr_kernel_launch_count.restype = i64
    L.lr_release_workspaces.argtypes = []
    for name in ("lr_linear", "lr_linear_f32", "lr_linear_strided", "lr_linear_group",
                 "lr_linear_host", "lr_dense",
                 "lr_linear_decode_static",
                 "lr_last_device_status", "lr_last_cuda_error", "lr_set_path",
                 "lr_set_wait_limit_ns", "lr_release_workspaces", "lr_set_withhold_first_stage",
                 "lr_set_tile_n", "lr_set_split_k", "lr_set_early_copy", "lr_gac_select",
                 "lr_set_t_precision"):
        getattr(L, name).restype = ctypes.c_int
    if path == LIB_PATH:
        _lib = L
    return L


def status_string(code: int) -> str:
    try:
        return lib().lr_status_string(code).decode()
    except Exception:
        return f"status {code}"


def _check(code: int, what: str):
    if code != LR_OK:
        raise LrError(code, what, lib().lr_last_cuda_error())


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check_bf16(name, t, shape=None):
    import torch
    if t is None:
        return
    if t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError(f"{name} must be a bf16 CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def lr_linear(X, A, B, bias=None, Y=None, stream=None):
    """Y = (X·A)·B + bias on the GPU (bf16 in/out, fp32 accumulation)."""
    import torch
    M, K = X.shape
    r = A.shape[1]
    N = B.shape[1]
    _check_bf16("X", X)
    _check_bf16("A", A, (K, r))
    _check_bf16("B", B, (r, N))
    _check_bf16("bias", bias, (N,))
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _check_bf16("Y", Y, (M, N))
    _check(lib().lr_linear(_ptr(X), _ptr(A), _ptr(B), _ptr(bias), _ptr(Y), M, K, r, N,
                           _stream_ptr(stream)), "lr_linear")
    return Y


def lr_linear_f32(X, A, B, bias=None, Y=None, stream=None):
    """Y = (X·A)·B + bias with Y in fp32 (the accumulator plus bias, not
    rounded to bf16); inputs bf16 as for lr_linear."""
    import torch
    M, K = X.shape
    r = A.shape[1]
    N = B.shape[1]
    _check_bf16("X", X)
    _check_bf16("A", A, (K, r))
    _check_bf16("B", B, (r, N))
    _check_bf16("bias", bias, (N,))
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
    if Y.dtype != torch.float32 or not Y.is_cuda or not Y.is_contiguous() or \
            tuple(Y.shape) != (M, N):
        raise TypeError("Y must be a contiguous fp32 CUDA tensor of shape (M, N)")
    _check(lib().lr_linear_f32(_ptr(X), _ptr(A), _ptr(B), _ptr(bias), _ptr(Y), M, K, r, N,
                               _stream_ptr(stream)), "lr_linear_f32")
    return Y


def lr_linear_strided(X, A, B, bias=None, Y=None, stream=None):
    """lr_linear on 2-D views with row strides (element stride 1): for
    instance a factor stored in a buffer of pitch lr_factor_pitch(r) and
    passed as buf[:, :r].  Y bf16 or fp32 (allocated bf16 if None)."""
    import torch
    M, K = X.shape
    r = A.shape[1]
    N = B.shape[1]
    for name, t in (("X", X), ("A", A), ("B", B)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or t.stride(1) != 1:
            raise TypeError(f"{name} must be a bf16 CUDA tensor with unit column stride")
    if A.shape[0] != K or B.shape[0] != r:
        raise ValueError("shapes do not chain")
    _check_bf16("bias", bias, (N,))
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    if Y.dtype not in (torch.bfloat16, torch.float32) or not Y.is_cuda or Y.stride(1) != 1 or \
            tuple(Y.shape) != (M, N):
        raise TypeError("Y must be a bf16 or fp32 CUDA tensor (M, N) with unit column stride")
    _check(lib().lr_linear_strided(_ptr(X), X.stride(0), _ptr(A), A.stride(0), _ptr(B),
                                   B.stride(0), _ptr(bias), _ptr(Y), Y.stride(0), M, K, r, N,
                                   1 if Y.dtype == torch.float32 else 0, _stream_ptr(stream)),
           "lr_linear_strided")
    return Y


def factor_pitch(cols: int) -> int:
    """Row pitch (elements) at which a stored factor is read in place."""
    return int(lib().lr_factor_pitch(int(cols)))


def prepare_factor(W):
    """A copy of the 2-D factor W stored at row pitch factor_pitch(cols) (a
    one-time copy when weights are loaded, not a step of a call), returned as
    the [rows, cols] view to pass to lr_linear_strided: its rows are read in
    place by every call, with no realignment copy."""
    import torch
    rows, cols = W.shape
    buf = torch.zeros((rows, factor_pitch(cols)), dtype=W.dtype, device=W.device)
    buf[:, :cols].copy_(W)
    return buf[:, :cols]


def lr_dense(X, W, bias=None, Y=None, stream=None):
    """Y = X·W + bias with the same kernels (the dense comparison)."""
    import torch
    M, K = X.shape
    N = W.shape[1]
    _check_bf16("X", X)
    _check_bf16("W", W, (K, N))
    _check_bf16("bias", bias, (N,))
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _check_bf16("Y", Y, (M, N))
    _check(lib().lr_dense(_ptr(X), _ptr(W), _ptr(bias), _ptr(Y), M, K, N, _stream_ptr(stream)),
           "lr_dense")
    return Y


def lr_linear_group(projs: Sequence[dict], M: int, stream=None):
    """Run several projections on the same M in one call.

    Each dict has X, A, B, Y (torch tensors or raw pointer ints), and
    optionally bias, ld_y (default N), K, r, N (taken from shapes when the
    entries are tensors) and y_f32 (Y is fp32; default: inferred from a Y
    tensor's dtype, else bf16).  Y may be a view into a packed buffer: pass
    the element pointer and ld_y explicitly via ``Y_ptr`` / ``ld_y``.
    ``silu_gate``: the list index of this projection's gate (its Y becomes
    silu(Y_gate) * its own product), or None.
    """
    import torch
    arr = (LrProj * max(1, len(projs)))()
    for i, p in enumerate(projs):
        A, B = p["A"], p["B"]
        K = p.get("K", A.shape[0] if hasattr(A, "shape") else None)
        r = p.get("r", A.shape[1] if hasattr(A, "shape") else None)
        N = p.get("N", B.shape[1] if hasattr(B, "shape") else None)
        y_ptr = p.get("Y_ptr", _ptr(p.get("Y")))
        y32 = p.get("y_f32", getattr(p.get("Y"), "dtype", None) == torch.float32)
        arr[i] = LrProj(_ptr(p["X"]) if hasattr(p["X"], "data_ptr") else p["X"], K,
                        _ptr(A) if hasattr(A, "data_ptr") else A,
                        _ptr(B) if hasattr(B, "data_ptr") else B,
                        _ptr(p.get("bias")) if hasattr(p.get("bias"), "data_ptr") else p.get("bias"),
                        y_ptr, p.get("ld_y", N), r, N, 1 if y32 else 0,
                        0 if p.get("silu_gate") is None else int(p["silu_gate"]) + 1)
    _check(lib().lr_linear_group(arr, len(projs), M, _stream_ptr(stream)), "lr_linear_group")


def lr_linear_host(X, A, B, bias=None, Y=None, stream=None):
    """The layer on HOST tensors (pinned or pageable): copies in, computes, copies out."""
    import torch
    M, K = X.shape
    r = A.shape[1]
    N = B.shape[1]
    for name, t in (("X", X), ("A", A), ("B", B), ("bias", bias)):
        if t is not None and (t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous()):
            raise TypeError(f"{name} must be a contiguous bf16 host tensor")
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, pin_memory=X.is_pinned())
    _check(lib().lr_linear_host(_ptr(X), _ptr(A), _ptr(B), _ptr(bias), _ptr(Y), M, K, r, N,
                                _stream_ptr(stream)), "lr_linear_host")
    return Y


def last_device_status(stream=None) -> int:
    return lib().lr_last_device_status(_stream_ptr(stream))


def set_path(path: int):
    _check(lib().lr_set_path(path), "lr_set_path")


def set_wait_limit_ns(ns: int):
    _check(lib().lr_set_wait_limit_ns(ns), "lr_set_wait_limit_ns")


def set_tile_n(bn: int):
    """Force the prefill tile width (32..256, multiple of 32); 0 = automatic."""
    _check(lib().lr_set_tile_n(bn), "lr_set_tile_n")


def set_split_k(on):
    """Split long K loops of small prefill GEMMs over several CTAs (True, the
    default) or not (False)."""
    _check(lib().lr_set_split_k(1 if on else 0), "lr_set_split_k")


def set_t_precision(mode: int):
    """How a prefill GEMM2 reads T: T_AUTO (0, the default), T_BF16 (1, T
    rounded once to bf16) or T_TWO_PARTS (2, T as bf16 hi + lo)."""
    _check(lib().lr_set_t_precision(int(mode)), "lr_set_t_precision")


def set_early_copy(on: bool):
    """Let a prefill call's realignment copy overlap the library's previous
    prefill launch on the stream (default on); off when the caller's own
    kernels between calls write operands and start their dependents early."""
    _check(lib().lr_set_early_copy(1 if on else 0), "lr_set_early_copy")


def gac_select(costs: Sequence[Sequence[int]], scores: Sequence[float],
               bases: Sequence[int], budget: int, unit: int):
    """lr_gac_select: one candidate index per weight (costs[i][j] parameters)
    maximising Σ scores[i]·(cost − bases[i]) within the quantized budget.
    Returns (choices, objective); raises LrError (LR_ERR_INFEASIBLE when
    nothing fits)."""
    n = len(costs)
    flat = [int(w) for c in costs for w in c]
    n_cand = (ctypes.c_int * max(n, 1))(*[len(c) for c in costs])
    cost = (ctypes.c_int64 * max(len(flat), 1))(*flat)
    score = (ctypes.c_double * max(n, 1))(*[float(s) for s in scores])
    base = (ctypes.c_int64 * max(n, 1))(*[int(b) for b in bases])
    choice = (ctypes.c_int * max(n, 1))()
    obj = ctypes.c_double()
    _check(lib().lr_gac_select(n, n_cand, cost, score, base, int(budget), int(unit), choice,
                               ctypes.byref(obj)), "lr_gac_select")
    return [int(c) for c in choice[:n]], obj.value


def set_withhold_first_stage(on: bool):
    """Testing failure detection: make the prefill kernels' bounded wait run out."""
    _check(lib().lr_set_withhold_first_stage(1 if on else 0), "lr_set_withhold_first_stage")


def kernel_launch_count() -> int:
    return int(lib().lr_kernel_launch_count())


def release_workspaces():
    _check(lib().lr_release_workspaces(), "lr_release_workspaces")

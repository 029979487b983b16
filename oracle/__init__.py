"""CPU fp64 oracle for Y = (X·A)·B (+bias) — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and, in ``bench.py``, the
CPU-baseline leg (which also checks 16 sampled GPU rows) and the reference
arm (``--impl reference``) may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and shares no code with
it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over output rows);
this module only builds it with gcc and marshals numpy arrays.  See the
header of ``oracle.c`` for the definition it computes and the passages it
follows ("Why Smaller Is Slower?", §1 and Figure 1; LowRankArena review,
"What SVD-based LLM compression actually does").

Pins (tests/test_oracle.py): exact rational arithmetic on tiny inputs,
associativity against a library matmul, identity and zero factors, and the
full-rank SVD invariant XAB = XW.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# -ffp-contract=off: no fused multiply-add, each product and sum is rounded
# once in fp64, as the plain definition states.  No -ffast-math.
CFLAGS = ["-O3", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off"]

_lib = None


def build(src: str = _SRC, out: str = _LIB, extra=()) -> str:
    """Compile oracle.c into a shared library (gcc)."""
    cmd = ["gcc", *CFLAGS, *extra, src, "-o", out]
    subprocess.run(cmd, check=True)
    return out


def load(path: str = _LIB):
    """Load (building first if needed) the oracle library and declare its ABI."""
    global _lib
    if path == _LIB and _lib is not None:
        return _lib
    if not os.path.exists(path) or (
        path == _LIB and os.path.getmtime(path) < os.path.getmtime(_SRC)
    ):
        build(out=path)
    lib = ctypes.CDLL(path)
    p = ctypes.c_void_p
    i64 = ctypes.c_int64
    lib.oracle_lr_linear.argtypes = [p, p, p, p, p, i64, i64, i64, i64, ctypes.c_int]
    lib.oracle_lr_linear_rows.argtypes = [p, p, p, p, p, i64, i64, i64, p, i64, ctypes.c_int]
    lib.oracle_lr_linear_f64.argtypes = [p, p, p, p, p, i64, i64, i64, i64, ctypes.c_int]
    lib.oracle_dense_rows.argtypes = [p, p, p, p, i64, i64, p, i64, ctypes.c_int]
    for f in (lib.oracle_lr_linear, lib.oracle_lr_linear_rows,
              lib.oracle_lr_linear_f64, lib.oracle_dense_rows):
        f.restype = ctypes.c_int
    if path == _LIB:
        _lib = lib
    return lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a, shape):
    if a is None:
        return None
    a = np.ascontiguousarray(a, dtype=np.uint16)
    assert a.shape == tuple(shape), (a.shape, shape)
    return a


def lr_linear(X, A, B, bias=None, rows=None, threads=None, lib=None) -> np.ndarray:
    """fp64 Y for bf16-bit inputs X [M,K], A [K,r], B [r,N], bias [N] or None.

    With ``rows`` (a sequence of row indices of X) only those output rows are
    computed; row i of the result is output row rows[i].
    """
    lib = lib or load()
    X = np.ascontiguousarray(X, dtype=np.uint16)
    M, K = X.shape
    r = np.asarray(A).shape[1] if np.asarray(A).ndim == 2 else 0
    N = np.asarray(B).shape[1]
    A = _u16(A, (K, r))
    B = _u16(B, (r, N))
    bias = _u16(bias, (N,))
    threads = threads or default_threads()
    if rows is None:
        Y = np.zeros((M, N), dtype=np.float64)
        rc = lib.oracle_lr_linear(_ptr(X), _ptr(A), _ptr(B), _ptr(bias), _ptr(Y),
                                  M, K, r, N, threads)
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        assert rows.size == 0 or (rows.min() >= 0 and rows.max() < M)
        Y = np.zeros((rows.size, N), dtype=np.float64)
        rc = lib.oracle_lr_linear_rows(_ptr(X), _ptr(A), _ptr(B), _ptr(bias), _ptr(Y),
                                       K, r, N, _ptr(rows), rows.size, threads)
    if rc != 0:
        raise RuntimeError("oracle failed (allocation or bad size)")
    return Y


def lr_linear_f64(X, A, B, bias=None, threads=None, lib=None) -> np.ndarray:
    """The same definition on fp64 inputs."""
    lib = lib or load()
    X = np.ascontiguousarray(X, dtype=np.float64)
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    M, K = X.shape
    r = A.shape[1]
    N = B.shape[1]
    assert A.shape == (K, r) and B.shape == (r, N)
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float64)
        assert bias.shape == (N,)
    Y = np.zeros((M, N), dtype=np.float64)
    rc = lib.oracle_lr_linear_f64(_ptr(X), _ptr(A), _ptr(B), _ptr(bias), _ptr(Y),
                                  M, K, r, N, threads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle failed")
    return Y


def dense(X, W, bias=None, rows=None, threads=None, lib=None) -> np.ndarray:
    """fp64 Y = X·W (+bias) for bf16-bit X [M,K], W [K,N] (listed rows only)."""
    lib = lib or load()
    X = np.ascontiguousarray(X, dtype=np.uint16)
    M, K = X.shape
    N = np.asarray(W).shape[1]
    W = _u16(W, (K, N))
    bias = _u16(bias, (N,))
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    Y = np.zeros((rows.size, N), dtype=np.float64)
    rc = lib.oracle_dense_rows(_ptr(X), _ptr(W), _ptr(bias), _ptr(Y), K, N,
                               _ptr(rows), rows.size, threads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle failed")
    return Y

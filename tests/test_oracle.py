"""Pins for the CPU fp64 oracle (no GPU).

Each pin checks the oracle against something other than itself:

* exact rational arithmetic (Python ``fractions``) on tiny odd-sized inputs,
  with the standard fp64 summation error bound;
* associativity: X·(A·B) through a library matmul, a different order;
* identity and zero factors, where the layer reduces to one GEMM or to the
  bias alone;
* the full-rank SVD invariant: with A = U·Σ and B = Vᵀ from an exact SVD of
  W, X·A·B equals X·W (Eckart–Young with k = min(m, n): the truncation is
  empty; LowRankArena review, "What SVD-based LLM compression actually does").

``test_pins_catch_planted_mistakes`` compiles altered copies of oracle.c
(a flipped sign, a dropped bias, a wrong stride, a short loop, fp32
accumulation, a shifted row) and checks that at least one pin rejects each.
"""
import os
import re
import shutil
from fractions import Fraction

import numpy as np
import pytest

import lrgen
import oracle

U = 2.0 ** -53


def _exact_lowrank(X, A, B, bias):
    """Exact rational Y and the elementwise |X||A||B| + |bias| magnitude."""
    Xf = [[Fraction(float(v)) for v in row] for row in lrgen.bf16_to_f64(X)]
    Af = [[Fraction(float(v)) for v in row] for row in lrgen.bf16_to_f64(A)]
    Bf = [[Fraction(float(v)) for v in row] for row in lrgen.bf16_to_f64(B)]
    bf = None if bias is None else [Fraction(float(v)) for v in lrgen.bf16_to_f64(bias)]
    M, K = len(Xf), len(Xf[0]) if Xf else 0
    r = A.shape[1]
    N = B.shape[1]
    Y = np.zeros((M, N))
    mag = np.zeros((M, N))
    for m in range(M):
        t = [sum((Xf[m][k] * Af[k][j] for k in range(K)), Fraction(0)) for j in range(r)]
        ta = [sum((abs(Xf[m][k] * Af[k][j]) for k in range(K)), Fraction(0)) for j in range(r)]
        for n in range(N):
            y = sum((t[j] * Bf[j][n] for j in range(r)), Fraction(0))
            ya = sum((ta[j] * abs(Bf[j][n]) for j in range(r)), Fraction(0))
            if bf is not None:
                y += bf[n]
                ya += abs(bf[n])
            Y[m, n] = float(y)
            mag[m, n] = float(ya)
    return Y, mag


TINY_SHAPES = [(1, 1, 1, 1), (3, 5, 7, 9), (5, 9, 3, 7), (2, 7, 9, 5), (4, 8, 1, 3), (5, 3, 5, 1)]


def pin_exact(lib):
    for s, (M, K, r, N) in enumerate(TINY_SHAPES):
        p = lrgen.lowrank_problem(M, K, r, N, seed=100 + s, bias=(s % 2 == 0))
        Y = oracle.lr_linear(p["X"], p["A"], p["B"], p["bias"], threads=1, lib=lib)
        Ye, mag = _exact_lowrank(p["X"], p["A"], p["B"], p["bias"])
        # |fl(Y) - Y| <= gamma_n · (|X||A||B| + |bias|), n = K + r + 1 terms deep.
        n = K + r + 2
        bound = (n * U / (1 - n * U)) * mag + 1e-300
        if not np.all(np.abs(Y - Ye) <= bound):
            return False
    return True


def pin_assoc(lib):
    for s, (M, K, r, N) in enumerate([(7, 33, 17, 29), (12, 64, 45, 31), (3, 20, 51, 8)]):
        p = lrgen.lowrank_problem(M, K, r, N, seed=200 + s, bias=True)
        Y = oracle.lr_linear(p["X"], p["A"], p["B"], p["bias"], lib=lib)
        X, A, B, b = (lrgen.bf16_to_f64(p[k]) for k in ("X", "A", "B", "bias"))
        ref = X @ (A @ B) + b[None, :]
        scale = np.linalg.norm(X) * np.linalg.norm(A) * np.linalg.norm(B) + np.abs(b).max()
        if not np.abs(Y - ref).max() <= 1e-12 * scale:
            return False
    return True


def _bf16_eye(n):
    return lrgen.bf16_bits(np.eye(n))


def pin_identity_zero(lib):
    M, K, N = 6, 13, 11
    p = lrgen.lowrank_problem(M, K, K, N, seed=300, bias=True)
    X, B, b = (lrgen.bf16_to_f64(p[k]) for k in ("X", "B", "bias"))
    # A = I (r = K): Y = X·B + bias.
    Y = oracle.lr_linear(p["X"], _bf16_eye(K), p["B"], p["bias"], lib=lib)
    if not np.allclose(Y, X @ B + b, rtol=0, atol=1e-13 * (np.abs(X) @ np.abs(B) + np.abs(b)).max()):
        return False
    # B = I (r = N): Y = X·A.
    q = lrgen.lowrank_problem(M, K, N, N, seed=301)
    Xq, Aq = lrgen.bf16_to_f64(q["X"]), lrgen.bf16_to_f64(q["A"])
    Y = oracle.lr_linear(q["X"], q["A"], _bf16_eye(N), None, lib=lib)
    if not np.allclose(Y, Xq @ Aq, rtol=0, atol=1e-13 * (np.abs(Xq) @ np.abs(Aq)).max()):
        return False
    # A = 0 or B = 0: Y = bias exactly.
    zA = np.zeros((K, 5), dtype=np.uint16)
    zB = np.zeros((5, N), dtype=np.uint16)
    rB = lrgen.lowrank_problem(M, K, 5, N, seed=302, bias=True)
    Y = oracle.lr_linear(rB["X"], zA, rB["B"], rB["bias"], lib=lib)
    if not np.array_equal(Y, np.broadcast_to(lrgen.bf16_to_f64(rB["bias"]), (M, N))):
        return False
    Y = oracle.lr_linear(rB["X"], rB["A"], zB, None, lib=lib)
    if not np.array_equal(Y, np.zeros((M, N))):
        return False
    return True


def pin_svd(lib):
    rng = np.random.default_rng(5)
    for (M, K, N) in [(9, 48, 40), (7, 31, 57)]:
        W = rng.standard_normal((K, N))
        X = rng.standard_normal((M, K))
        Uw, S, Vt = np.linalg.svd(W, full_matrices=False)
        A = Uw * S[None, :]
        Y = oracle.lr_linear_f64(X, A, Vt, lib=lib)
        if not np.abs(Y - X @ W).max() <= 1e-10:
            return False
    return True


PINS = [pin_exact, pin_assoc, pin_identity_zero, pin_svd]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    assert pin(oracle.load())


def test_rows_subset_matches_full():
    p = lrgen.lowrank_problem(37, 70, 23, 45, seed=11, bias=True)
    Y = oracle.lr_linear(p["X"], p["A"], p["B"], p["bias"])
    rows = [36, 0, 17, 17, 5]
    Ys = oracle.lr_linear(p["X"], p["A"], p["B"], p["bias"], rows=rows)
    assert np.array_equal(Ys, Y[rows])


def test_empty_sizes():
    # r = 0 or K = 0: the empty sum is 0, so Y = bias (or 0).
    p = lrgen.lowrank_problem(4, 6, 0, 5, seed=1, bias=True)
    Y = oracle.lr_linear(p["X"], np.zeros((6, 0), np.uint16), np.zeros((0, 5), np.uint16), p["bias"])
    assert np.array_equal(Y, np.broadcast_to(lrgen.bf16_to_f64(p["bias"]), (4, 5)))
    Y = oracle.lr_linear(np.zeros((4, 0), np.uint16), np.zeros((0, 3), np.uint16),
                         lrgen.normal_bf16(1, 3, (3, 5)), None)
    assert np.array_equal(Y, np.zeros((4, 5)))
    Y = oracle.lr_linear(np.zeros((0, 6), np.uint16), lrgen.normal_bf16(1, 2, (6, 3)),
                         lrgen.normal_bf16(1, 3, (3, 5)), None)
    assert Y.shape == (0, 5)


def test_dense_oracle_matches_lowrank_with_identity():
    # X·W through the dense oracle equals the low-rank oracle with A = W, B = I.
    p = lrgen.lowrank_problem(5, 19, 13, 13, seed=12, bias=True)
    Yd = oracle.dense(p["X"], p["A"], p["bias"])
    Yl = oracle.lr_linear(p["X"], p["A"], _bf16_eye(13), p["bias"])
    assert np.abs(Yd - Yl).max() <= 1e-14 * max(1.0, np.abs(Yd).max())


def test_rms_of_fan_in_scaled_layer_is_near_one():
    # X ~ N(0,1), A ~ N(0,1/K), B ~ N(0,1/r): E[Y²] = 1.
    p = lrgen.lowrank_problem(16, 256, 107, 256, seed=0)
    Y = oracle.lr_linear(p["X"], p["A"], p["B"])
    rms = np.sqrt(np.mean(Y ** 2))
    assert 0.85 < rms < 1.15


# (pattern, replacement) pairs: each is one plausible slip in the oracle.
MUTANTS = {
    "sign_T": (r"t\[j\] \+= xk \* a\[j\];", "t[j] -= xk * a[j];"),
    "drop_bias": (r"Yrow\[n\] \+= b\[n\];", "Yrow[n] += 0.0 * b[n];"),
    "B_stride": (r"f\(B, j, N, N, b\);", "f(B, j, N, r, b);"),
    "A_stride": (r"f\(A, k, r, r, a\);", "f(A, k, r, K, a);"),
    "short_r": (r"for \(int64_t j = 0; j < r; \+\+j\) \{", "for (int64_t j = 0; j + 1 < r; ++j) {"),
    "fp32_T": (r"t\[j\] \+= xk \* a\[j\];", "t[j] = (float)(t[j] + xk * a[j]);"),
    "row_shift": (r"f\(X, m, K, K, x\);", "f(X, m > 0 ? m - 1 : 0, K, K, x);"),
    "transpose_B": (r"f\(B, j, N, N, b\);",
                    "for (int64_t q = 0; q < N; ++q) b[q] = (q < r && j < N) ? "
                    "bf16_value(((const uint16_t *)B)[q * N + j]) : 0.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    pat, rep = MUTANTS[name]
    mutated, n = re.subn(pat, rep, src, count=1)
    assert n == 1, f"mutation {name} did not apply"
    cpath = tmp_path / "oracle_mut.c"
    cpath.write_text(mutated)
    so = str(tmp_path / "liboracle_mut.so")
    oracle.build(src=str(cpath), out=so)
    lib = oracle.load(so)
    results = {}
    for pin in PINS:
        try:
            results[pin.__name__] = bool(pin(lib))
        except Exception:
            results[pin.__name__] = False
    assert not all(results.values()), f"no pin caught mutant {name}: {results}"

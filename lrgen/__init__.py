"""Seeded synthetic inputs for the low-rank linear layer Y = (X·A)·B (+bias).

This module is shared by the tests, the bench and the oracle checks.  It holds
no arithmetic of the layer itself: it only draws numbers and rounds them to
bf16.  Everything it returns is a numpy ``uint16`` array of bf16 bit patterns
(row-major), so the CPU oracle and the GPU path read exactly the same bits.

Random numbers
--------------
A counter-based generator: SplitMix64 (Steele, Lea, Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014) applied to the counter
``key + (i+1)·0x9E3779B97F4A7C15``, where ``key`` is derived from the
``(seed, tensor_id)`` pair and ``i`` is the element's counter.  Uniforms are the
top 53 bits, offset by half an ulp so they lie in (0, 1).  Normals use the
Box–Muller transform on the uniforms of counters 2i and 2i+1.  Every value is
drawn in fp64 and rounded once, to nearest-even, into bf16.

Workload shapes
---------------
The shapes follow the Llama-3-8B projections the pages measure on (GAC paper
§5.1; LowRankArena review, keep-ratio worked example).  No model weights or
dataset items are used: factors are N(0, 1/fan_in) draws, and the prefill
q_proj case builds A = U·Σ and B = Vᵀ from Haar-orthogonal U, V with
σ_i = i^-0.5 (LowRankArena review, "What SVD-based LLM compression actually
does", Eckart–Young truncation).
"""
from __future__ import annotations

import math
import numpy as np

__all__ = [
    "GAMMA", "splitmix64", "uniform", "normal", "bf16_bits", "bf16_to_f64",
    "normal_bf16", "lowrank_problem", "svd_problem", "haar_orthogonal",
    "decoder_layer", "LAYER_PROJECTIONS", "TENSOR_ID",
]

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Fixed stream ids per tensor role, so that one tensor's values never depend
# on which other tensors were drawn before it.
TENSOR_ID = {"X": 1, "A": 2, "B": 3, "bias": 4, "GU": 10, "GV": 11, "W": 12}


def splitmix64(z: np.ndarray) -> np.ndarray:
    """The SplitMix64 finaliser on a uint64 array (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int, tensor_id: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = splitmix64(np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64) + GAMMA)
        k = splitmix64(s ^ np.uint64(tensor_id & 0xFFFFFFFFFFFFFFFF))
    return k[0]


def _bits(seed: int, tensor_id: int, counters: np.ndarray) -> np.ndarray:
    key = _key(seed, tensor_id)
    with np.errstate(over="ignore"):
        z = key + (counters.astype(np.uint64) + np.uint64(1)) * GAMMA
    return splitmix64(z)


def uniform(seed: int, tensor_id: int, counters: np.ndarray) -> np.ndarray:
    """Uniform fp64 values in (0, 1) for the given counters."""
    b = _bits(seed, tensor_id, counters)
    return ((b >> np.uint64(11)).astype(np.float64) + 0.5) * (1.0 / 9007199254740992.0)


def normal(seed: int, tensor_id: int, n: int, start: int = 0) -> np.ndarray:
    """n standard-normal fp64 draws for element counters start .. start+n-1."""
    out = np.empty(n, dtype=np.float64)
    chunk = 1 << 22
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        i = np.arange(start + lo, start + hi, dtype=np.uint64)
        u1 = uniform(seed, tensor_id, np.uint64(2) * i)
        u2 = uniform(seed, tensor_id, np.uint64(2) * i + np.uint64(1))
        out[lo:hi] = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)
    return out


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (nearest, ties to even) and return the bits.

    The value is rounded once, directly from fp64 (no fp32 step, so no double
    rounding).  Magnitudes below 2^-120 are flushed to a signed zero; the
    distributions used here never reach them.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m·2^e, 0.5 <= |m| < 1
    q = np.rint(m * 256.0)                  # 8 significant bits, ties to even
    y = np.ldexp(q, e - 8)
    y = np.where(np.abs(x) < 2.0 ** -120, np.copysign(0.0, x), y)
    if not np.all(np.isfinite(y)) or np.any(np.abs(y) >= 2.0 ** 127):
        raise ValueError("value outside the bf16 range used by the generator")
    f = y.astype(np.float32)                # exact: y has <= 8 significant bits
    u = f.view(np.uint32)
    assert not np.any(u & np.uint32(0xFFFF)), "bf16 rounding left low bits"
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp64 (exact)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return u.view(np.float32).astype(np.float64)


def normal_bf16(seed: int, tensor_id: int, shape, std: float = 1.0, row0: int = 0) -> np.ndarray:
    """bf16 bits of N(0, std²) draws with the given shape (row-major counters).

    ``row0``: the rows row0 .. row0 + shape[0] - 1 of a taller matrix with the
    same columns (its counters start at row0·cols), so that row blocks drawn
    separately (one per rank of a data-parallel batch) are the matching rows
    of the matrix drawn whole.
    """
    n = int(np.prod(shape)) if len(shape) else 1
    cols = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    return bf16_bits(normal(seed, tensor_id, n, start=row0 * cols) * std).reshape(shape)


def lowrank_problem(M: int, K: int, r: int, N: int, seed: int = 0,
                    bias: bool = False, tid_base: int = 0) -> dict:
    """X ~ N(0,1) [M,K]; A ~ N(0,1/K) [K,r]; B ~ N(0,1/r) [r,N]; bias ~ N(0,1) [N].

    "N(0, 1/fan_in)" is read as variance 1/fan_in, with fan_in(A) = K and
    fan_in(B) = r.  ``tid_base`` offsets the stream ids so that several
    projections drawn with one seed stay independent.
    """
    t = TENSOR_ID
    out = {
        "M": M, "K": K, "r": r, "N": N,
        "X": normal_bf16(seed, tid_base + t["X"], (M, K), 1.0),
        "A": normal_bf16(seed, tid_base + t["A"], (K, r), 1.0 / math.sqrt(K) if K else 1.0),
        "B": normal_bf16(seed, tid_base + t["B"], (r, N), 1.0 / math.sqrt(r) if r else 1.0),
        "bias": normal_bf16(seed, tid_base + t["bias"], (N,), 1.0) if bias else None,
    }
    return out


def haar_orthogonal(seed: int, tensor_id: int, n: int) -> np.ndarray:
    """A Haar-distributed n×n orthogonal matrix (fp64).

    Q·diag(sign(diag R)) from the Householder QR of an n×n N(0,1) matrix has
    the Haar distribution (Mezzadri, "How to generate random matrices from the
    classical compact groups", Notices AMS 2007), the same law as the singular
    vectors of a Gaussian matrix.
    """
    G = normal(seed, tensor_id, n * n).reshape(n, n)
    Q, R = np.linalg.qr(G)
    s = np.sign(np.diag(R))
    s[s == 0] = 1.0
    return Q * s[None, :]


def svd_problem(M: int = 2048, K: int = 4096, N: int = 4096, r: int = 1741,
                seed: int = 0, keep_f64: bool = False) -> dict:
    """Prefill q_proj case: A = U[:, :r]·diag(σ), B = V[:, :r]ᵀ, σ_i = i^-0.5.

    W [K,N] = U·Σ·Vᵀ is never formed.  U and V are Haar orthogonal; all of Σ
    goes into A (the factor convention of the workload definition; the pages'
    split of Σ^1/2 into both factors gives the same product).  A and B are
    rounded to bf16 only after the fp64 products.
    """
    U = haar_orthogonal(seed, TENSOR_ID["GU"], K)
    V = haar_orthogonal(seed, TENSOR_ID["GV"], N)
    n_sig = min(K, N)
    sigma = np.arange(1, n_sig + 1, dtype=np.float64) ** -0.5
    A64 = U[:, :r] * sigma[None, :r]
    B64 = np.ascontiguousarray(V[:, :r].T)
    out = {
        "M": M, "K": K, "r": r, "N": N,
        "X": normal_bf16(seed, TENSOR_ID["X"], (M, K), 1.0),
        "A": bf16_bits(A64),
        "B": bf16_bits(B64),
        "bias": None,
        "sigma": sigma,
    }
    if keep_f64:
        out.update(U=U, V=V, A64=A64, B64=B64)
    return out


# Llama-3-8B decoder-layer projections: (name, K, N, X-sharing set).
LAYER_PROJECTIONS = [
    ("q", 4096, 4096, "attn_in"),
    ("k", 4096, 1024, "attn_in"),
    ("v", 4096, 1024, "attn_in"),
    ("o", 4096, 4096, "o_in"),
    ("gate", 4096, 14336, "mlp_in"),
    ("up", 4096, 14336, "mlp_in"),
    ("down", 14336, 4096, "down_in"),
]


def layer_ranks(seed: int = 7, n_int: int = 14336) -> dict:
    """Per-projection ranks: integers uniform on [ceil(0.35·m), floor(0.85·m)],
    m = min(K, N), drawn in the order q, k, v, o, gate, up, down from one
    counter stream of ``seed``.  Ranks are left as drawn (not snapped to 8)."""
    ranks = {}
    for idx, (name, K, N, _) in enumerate(LAYER_PROJECTIONS):
        if name in ("gate", "up"):
            N = n_int
        if name == "down":
            K = n_int
        m = min(K, N)
        lo, hi = math.ceil(0.35 * m), math.floor(0.85 * m)
        u = uniform(seed, 900, np.array([idx], dtype=np.uint64))[0]
        ranks[name] = lo + int(u * (hi - lo + 1))
    return ranks


def decoder_layer(M: int, seed: int = 7, n_int: int = 14336, bias: bool = False) -> dict:
    """A factorized decoder layer: per-projection factors and shared inputs.

    gate and up are separate factor pairs that share X and write into one
    packed Y of width 2·n_int; down reads K = n_int.  Returns a dict with
    "inputs" (one X per sharing set) and "projs" (name → problem dict with
    "x" naming its input).
    """
    ranks = layer_ranks(seed, n_int)
    inputs = {}
    projs = {}
    for idx, (name, K, N, xset) in enumerate(LAYER_PROJECTIONS):
        if name in ("gate", "up"):
            N = n_int
        if name == "down":
            K = n_int
        if xset not in inputs:
            tid = 5000 + 10 * len(inputs)
            inputs[xset] = normal_bf16(seed, tid, (M, K), 1.0)
        r = ranks[name]
        base = 100 * (idx + 1)
        p = {
            "name": name, "x": xset, "M": M, "K": K, "r": r, "N": N,
            "A": normal_bf16(seed, base + TENSOR_ID["A"], (K, r), 1.0 / math.sqrt(K)),
            "B": normal_bf16(seed, base + TENSOR_ID["B"], (r, N), 1.0 / math.sqrt(r)),
            "bias": normal_bf16(seed, base + TENSOR_ID["bias"], (N,), 1.0) if bias else None,
        }
        projs[name] = p
    return {"M": M, "inputs": inputs, "projs": projs, "ranks": ranks, "n_int": n_int}


def gac_model(layers: int = 32, seed: int = 11, n_int: int = 14336) -> list:
    """Inputs for GAC's rank re-selection over `layers` decoder layers of the
    Llama-3-8B projection shapes: per weight an unconstrained (fractional)
    rank r* uniform on [0.35·m, 0.85·m], m = min(K, N), and an importance
    score uniform on [0.5, 1.5), drawn weight by weight from counter streams
    of ``seed`` (these stand in for a compressor's allocation and its
    importance scores, which need trained weights)."""
    out = []
    idx = 0
    for layer in range(layers):
        for name, K, N, _ in LAYER_PROJECTIONS:
            if name in ("gate", "up"):
                N = n_int
            if name == "down":
                K = n_int
            m = min(K, N)
            c = np.array([idx], dtype=np.uint64)
            u = uniform(seed, 901, c)[0]
            s = uniform(seed, 902, c)[0]
            out.append({"name": f"layers.{layer}.{name}", "K": K, "N": N,
                        "r_star": float((0.35 + 0.5 * u) * m), "score": float(0.5 + s)})
            idx += 1
    return out

"""Host-side accounting for the low-rank linear layer: parameter counts, keep
ratio, algorithmic FLOPs and bytes, and the roofline time they imply.

Nothing here runs on the GPU; the bench and the tests use it.

* Parameter count of a rank-k factorisation of an m×n weight: k(m+n) instead
  of mn (LowRankArena review, "What SVD-based LLM compression actually does").
* Keep ratio over a set of layers: the sum of the factorised parameter counts
  over the sum of the dense counts, at equal precision (LowRankArena review,
  "The standardized keep-ratio formula, expanded"; worked example in
  "A worked numerical example of the keep-ratio formula": 0.636).
* Algorithmic work of Y = (X·A)·B: 2·M·r·(K+N) FLOPs and (MK+Kr+rN+MN)·2
  bytes for bf16 tensors.  The intermediate T's round trip, padding and any
  recompute are not algorithmic and are excluded.
* Break-even rank against the dense layer: r·(K+N) < K·N, i.e.
  r < K·N/(K+N) (the dense fallback the LowRankArena review describes for
  DoBi-SVD, Q3).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Iterable, Sequence

BF16_BYTES = 2


def lowrank_params(m: int, n: int, k: int) -> int:
    """Stored scalars of a rank-k factorisation of an m×n matrix: k(m+n)."""
    if min(m, n, k) < 0:
        raise ValueError("negative size")
    return k * (m + n)


def dense_params(m: int, n: int) -> int:
    return m * n


def keep_ratio(layers: Iterable[Sequence[int]]) -> float:
    """Keep ratio of (m, n, k) layers: Σ k(m+n) / Σ mn (sum, then divide)."""
    num = 0
    den = 0
    for m, n, k in layers:
        num += lowrank_params(m, n, k)
        den += dense_params(m, n)
    if den == 0:
        raise ValueError("no layers")
    return num / den


def keep_ratio_terms(layers: Iterable[Sequence[int]]) -> tuple[int, int]:
    """(numerator, denominator) of the keep ratio, as exact integers."""
    num = 0
    den = 0
    for m, n, k in layers:
        num += lowrank_params(m, n, k)
        den += dense_params(m, n)
    return num, den


def break_even_rank(K: int, N: int) -> float:
    """Rank above which the factorised layer stores (and streams) more than W."""
    return K * N / (K + N)


def flops(M: int, K: int, r: int, N: int) -> int:
    """2·M·r·(K+N): both contractions, one multiply and one add per term."""
    return 2 * M * r * (K + N)


def dense_flops(M: int, K: int, N: int) -> int:
    return 2 * M * K * N


def algorithmic_bytes(M: int, K: int, r: int, N: int, bias: bool = False,
                      count_x: bool = True) -> int:
    """(MK + Kr + rN + MN)·2 (+ N·2 for a bias): each tensor read or written once."""
    b = (K * r + r * N + M * N) * BF16_BYTES
    if count_x:
        b += M * K * BF16_BYTES
    if bias:
        b += N * BF16_BYTES
    return b


def dense_bytes(M: int, K: int, N: int) -> int:
    return (M * K + K * N + M * N) * BF16_BYTES


@dataclass(frozen=True)
class Roofline:
    flops: int
    bytes: int
    t_compute_s: float
    t_memory_s: float

    @property
    def t_roof_s(self) -> float:
        return max(self.t_compute_s, self.t_memory_s)

    @property
    def bound(self) -> str:
        return "tensor" if self.t_compute_s >= self.t_memory_s else "hbm"


def roofline(fl: int, by: int, peak_tflops: float, peak_gbs: float) -> Roofline:
    """Roofline time: the slower of FLOPs at the tensor peak and bytes at HBM peak."""
    return Roofline(fl, by, fl / (peak_tflops * 1e12), by / (peak_gbs * 1e9))


def group_work(M: int, projs: Sequence[dict]) -> tuple[int, int]:
    """FLOPs and algorithmic bytes of a projection group.

    Each dict has K, r, N and an "x" key naming its input; an input shared by
    several projections is counted once.
    """
    fl = 0
    by = 0
    seen = set()
    for p in projs:
        fl += flops(M, p["K"], p["r"], p["N"])
        first = p["x"] not in seen
        seen.add(p["x"])
        by += algorithmic_bytes(M, p["K"], p["r"], p["N"], bias=p.get("bias") is not None,
                                count_x=first)
    return fl, by

"""GAC's alignment-aware re-selection of compressed ranks (host side).

"Why Smaller Is Slower? Dimensional Misalignment in Compressed LLMs", §4
GAC: GPU-Aligned Compression.  Step 1, the compressor's unconstrained
allocation r_i*, happens upstream.  Step 2, the dimension sweep (§4.2),
proposes aligned ranks near r_i* (``sweep_ranks``) and keeps those whose
measured time on this GPU shows no cliff (``drop_cliffs``; the times come
from timing lr_linear at each rank, as ``bench.py --gac-sweep`` does).  Step 3
(§4.3) picks one candidate per weight under the same parameter budget
(``plan``, which calls lr_gac_select in the C library).

A rank whose factorisation stores at least as many parameters as the dense
weight (r·(K+N) ≥ K·N) is replaced by the dense weight itself, the dense
fallback the LowRankArena review describes for DoBi-SVD.

    python -m rank_linear_layers_b200.gac     # plans a 32-layer model, times it
    python bench.py --gac-sweep > sweep.json  # per-shape rank timings on the GPU
    python -m rank_linear_layers_b200.gac --times sweep.json
"""
from __future__ import annotations

import math
import time
from dataclasses import dataclass
from typing import Mapping, Optional, Sequence

from . import gac_select

#: rank value of the dense-fallback candidate
DENSE = None


@dataclass(frozen=True)
class Weight:
    """One compressed weight W [K, N] ≈ A [K, r] · B [r, N]."""
    name: str
    K: int
    N: int
    r_star: float       # the compressor's unconstrained rank
    score: float = 1.0  # importance s_i

    @property
    def step_cost(self) -> int:
        """Parameters one unit of rank costs: K + N."""
        return self.K + self.N

    @property
    def dense_cost(self) -> int:
        return self.K * self.N


@dataclass
class Plan:
    ranks: dict          # name -> chosen rank (DENSE for the dense weight)
    params: dict         # name -> stored parameters
    total_params: int
    budget: int
    unit: int
    objective: float
    aligned_fraction: float


def sweep_ranks(r_star: float, align: int = 8, coarse: int = 4,
                limit: Optional[int] = None) -> list:
    """Aligned ranks near r_star: the multiples of `align` within 1.5·align
    of r_star, and the first multiple of coarse·align at or above it (the
    stricter alignments the paper's constraint table rewards).  For
    r* = 107.3 this is {96, 104, 112, 128}, the set §4.2's example lists.
    Ranks above `limit` (min(K, N)) are left out."""
    if align < 1 or coarse < 1 or not r_star > 0:
        raise ValueError("align, coarse and r_star must be positive")
    lo = max(align, math.ceil((r_star - 1.5 * align) / align) * align)
    hi = math.floor((r_star + 1.5 * align) / align) * align
    out = set(range(lo, hi + 1, align))
    big = coarse * align
    out.add(max(big, math.ceil(r_star / big) * big))
    if limit is not None:
        out = {d for d in out if d <= limit}
    return sorted(out)


def drop_cliffs(ranks: Sequence[int], times: Mapping[int, float], tol: float = 0.05) -> list:
    """Keep a rank unless a larger rank of the sweep ran faster by more than
    `tol` (a performance cliff: fewer parameters, more time).  Ranks without
    a measured time are kept."""
    kept = []
    for d in ranks:
        t = times.get(d)
        if t is not None and any(times.get(e) is not None and times[e] * (1.0 + tol) < t
                                 for e in ranks if e > d):
            continue
        kept.append(d)
    return kept


def candidates(w: Weight, times: Optional[Mapping[int, float]] = None, align: int = 8,
               coarse: int = 4, tol: float = 0.05) -> list:
    """(rank, parameters) candidates of one weight: the swept ranks without
    cliffs, ranks at or past the break-even r·(K+N) ≥ K·N replaced by one
    dense candidate (rank DENSE, K·N parameters)."""
    ranks = sweep_ranks(w.r_star, align, coarse, limit=min(w.K, w.N))
    if times:
        ranks = drop_cliffs(ranks, times, tol)
    out, dense = [], False
    for d in ranks:
        c = d * w.step_cost
        if c >= w.dense_cost:
            dense = True
        else:
            out.append((d, c))
    if dense or not out:
        out.append((DENSE, w.dense_cost))
    return out


def sweep_plan(weights: Sequence[Weight], align: int = 8, coarse: int = 4) -> dict:
    """The ranks to time for each weight shape: {(K, N): sorted ranks}, the
    union of the weights' swept ranks (one timing serves every weight of a
    shape)."""
    plan = {}
    for w in weights:
        plan.setdefault((w.K, w.N), set()).update(
            sweep_ranks(w.r_star, align, coarse, limit=min(w.K, w.N)))
    return {k: sorted(v) for k, v in plan.items()}


def times_by_weight(weights: Sequence[Weight], shape_times: Mapping) -> dict:
    """Per-weight rank timings from per-shape ones.  `shape_times` maps
    "KxN" (as ``bench.py --gac-sweep`` writes it) or (K, N) to {rank: time}."""
    out = {}
    for w in weights:
        t = shape_times.get(f"{w.K}x{w.N}", shape_times.get((w.K, w.N)))
        if t:
            out[w.name] = {int(r): float(v) for r, v in t.items()}
    return out


def budget_for(weights: Sequence[Weight]) -> int:
    """The compressor's own budget: Σ r_i*·(K_i + N_i), rounded down (GAC
    re-selects under the same parameter budget)."""
    return int(math.floor(sum(w.r_star * w.step_cost for w in weights)))


def plan(weights: Sequence[Weight], budget: Optional[int] = None,
         times: Optional[Mapping[str, Mapping[int, float]]] = None, align: int = 8,
         coarse: int = 4, tol: float = 0.05) -> Plan:
    """Step 3: one candidate per weight maximising Σ s_i·(|W_i| − |W_i*|)
    with Σ |W_i| ≤ budget, costs quantized by u = align·min_i (K_i + N_i)."""
    if not weights:
        raise ValueError("no weights")
    if budget is None:
        budget = budget_for(weights)
    cands = [candidates(w, (times or {}).get(w.name), align, coarse, tol) for w in weights]
    unit = align * min(w.step_cost for w in weights)
    costs = [[c for _, c in cs] for cs in cands]
    bases = [int(round(w.r_star * w.step_cost)) for w in weights]
    choice, obj = gac_select(costs, [w.score for w in weights], bases, budget, unit)
    ranks = {w.name: cands[i][j][0] for i, (w, j) in enumerate(zip(weights, choice))}
    params = {w.name: cands[i][j][1] for i, (w, j) in enumerate(zip(weights, choice))}
    aligned = sum(1 for r in ranks.values() if r is DENSE or r % align == 0)
    return Plan(ranks=ranks, params=params, total_params=sum(params.values()), budget=int(budget),
                unit=unit, objective=obj, aligned_fraction=aligned / len(weights))


def _main() -> int:
    import argparse
    import json

    import lrgen
    ap = argparse.ArgumentParser(description="Plan GAC ranks for a Llama-3-8B-shaped model")
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--seed", type=int, default=11)
    ap.add_argument("--repeat", type=int, default=5)
    ap.add_argument("--times", help="JSON written by `bench.py --gac-sweep` (per-shape rank timings)")
    ap.add_argument("--tol", type=float, default=0.05)
    args = ap.parse_args()
    ws = [Weight(**d) for d in lrgen.gac_model(args.layers, args.seed)]
    wt = None
    if args.times:
        with open(args.times) as f:
            wt = times_by_weight(ws, json.load(f)["times_us"])
    times = []
    for _ in range(args.repeat):
        t0 = time.perf_counter()
        p = plan(ws, times=wt, tol=args.tol)
        times.append(time.perf_counter() - t0)
    cliffs = 0
    if wt:
        for w in ws:
            swept = sweep_ranks(w.r_star, limit=min(w.K, w.N))
            cliffs += len(swept) - len(drop_cliffs(swept, wt.get(w.name, {}), args.tol))
    unaligned = sum(1 for w in ws if abs(w.r_star - round(w.r_star)) > 0 or round(w.r_star) % 8)
    print(json.dumps({
        "weights": len(ws), "budget": p.budget, "unit": p.unit,
        "quantized_budget": p.budget // p.unit, "total_params": p.total_params,
        "objective": p.objective, "aligned_fraction": p.aligned_fraction,
        "unaligned_before": unaligned / len(ws),
        "dense_fallbacks": sum(1 for r in p.ranks.values() if r is DENSE),
        "measured_times": bool(wt), "cliffs_dropped": cliffs,
        "plan_ms_median": sorted(times)[len(times) // 2] * 1e3}))
    return 0


if __name__ == "__main__":
    raise SystemExit(_main())

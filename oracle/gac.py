"""Plain reference of GAC's constrained re-selection of dimensions — TEST
INFRASTRUCTURE ONLY (imported by ``tests/`` alone; the product path never
uses it and shares no code with it).

Follows "Why Smaller Is Slower? Dimensional Misalignment in Compressed LLMs",
§4.3 Step 3: Constrained Optimization: pick one candidate dimension d_i ∈ C_i
per compressed weight to maximise Σ_i s_i·(|W_i| − |W_i*|) subject to
Σ_i |W_i| ≤ B, solved as a multiple-choice knapsack with the recurrence
D[i][b] = max_j D[i−1][b − w_ij] + v_ij, after the budget quantization of the
same section (costs and budget divided by a unit u = 8·M_min).

Readings where the section is silent:
* D[0][b] = 0 for every b ≥ 0, so D[n][B'] is the best selection of total
  quantized cost at most B' (the constraint is an inequality).
* Quantized costs are rounded up and the quantized budget down
  (w'_ij = ⌈w_ij/u⌉, B' = ⌊B/u⌋): every selection the table admits then
  satisfies the unquantized budget, the guarantee the paper claims.
* v_ij = s_i·(w_ij − |W_i*|) in fp64, accumulated over the weights in order.
* Ties: for each weight and remaining budget the lowest candidate index is
  kept (any optimum is correct; this one is unique and reproducible).

Pins (tests/test_gac.py): exhaustive enumeration of every selection on tiny
problems (exact integer arithmetic), closed-form cases (ample budget, budget
equal to the cheapest selection, one upgrade between two weights), the
budget-quantization example the section prints (u = 8·1024 for 1024-row
matrices), and the budget guarantee on random problems.
"""
from __future__ import annotations

import itertools
from typing import Optional, Sequence

import numpy as np


def quantize(costs: Sequence[Sequence[int]], budget: int, unit: int):
    """w'_ij = ⌈w_ij / u⌉ and B' = ⌊B / u⌋ (integers)."""
    if unit < 1 or budget < 0:
        raise ValueError("unit must be >= 1 and budget >= 0")
    wq = [[-(-int(w) // unit) for w in c] for c in costs]
    return wq, int(budget) // unit


def select(costs: Sequence[Sequence[int]], scores: Sequence[float], bases: Sequence[int],
           budget: int, unit: int) -> Optional[tuple[list[int], float]]:
    """The recurrence of §4.3 on the quantized costs: (choices, objective),
    or None when no selection fits the budget."""
    wq, bq = quantize(costs, budget, unit)
    D = np.zeros(bq + 1)  # D[0][b] = 0
    args = []
    for i, c in enumerate(costs):
        rows = np.full((len(c), bq + 1), -np.inf)
        for j, w in enumerate(c):
            v = float(scores[i]) * float(int(w) - int(bases[i]))
            k = wq[i][j]
            if k <= bq:
                rows[j, k:] = D[:bq + 1 - k] + v  # D[i-1][b - w'_ij] + v_ij
        a = np.argmax(rows, axis=0)  # first index of the maximum
        D = rows[a, np.arange(bq + 1)]
        args.append(a)
    if not D[bq] > -np.inf:
        return None
    choices = [0] * len(costs)
    b = bq
    for i in range(len(costs) - 1, -1, -1):
        j = int(args[i][b])
        choices[i] = j
        b -= wq[i][j]
    return choices, float(D[bq])


def objective(costs, scores, bases, choices) -> float:
    """Σ_i s_i·(w_i,choice − |W_i*|), summed over the weights in order."""
    total = 0.0
    for i, j in enumerate(choices):
        total = total + float(scores[i]) * float(int(costs[i][j]) - int(bases[i]))
    return total


def brute_force(costs, scores, bases, budget: int, unit: int):
    """Every selection enumerated: (best objective, [all optimal choice
    lists]) over those whose quantized cost fits, or (None, []) if none fits.
    Exact for integer scores and costs (small problems only)."""
    wq, bq = quantize(costs, budget, unit)
    best, arg = None, []
    for sel in itertools.product(*[range(len(c)) for c in costs]):
        if sum(wq[i][j] for i, j in enumerate(sel)) > bq:
            continue
        val = sum(scores[i] * (costs[i][j] - bases[i]) for i, j in enumerate(sel))
        if best is None or val > best:
            best, arg = val, [list(sel)]
        elif val == best:
            arg.append(list(sel))
    return best, arg

"""GAC's constrained re-selection of dimensions ("Why Smaller Is Slower?",
§4.2 Dimension Sweep and §4.3 Constrained Optimization): the plain oracle
against its pins, the C solver (lr_gac_select) against the oracle, and the
host logic that builds candidate sets.  No GPU needed."""
import ctypes
import math
import os
import random

import numpy as np
import pytest

import lrgen
import rank_linear_layers_b200 as lr
from oracle import gac as ref
from rank_linear_layers_b200 import gac

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def L():
    from rank_linear_layers_b200 import build
    if build.needs_build():
        build.build()
    return lr.lib()


def random_problem(rng, n_max=4, m_max=4, cost_max=40, integer=True):
    n = rng.randint(1, n_max)
    costs = [sorted(rng.sample(range(0, cost_max), rng.randint(1, m_max))) for _ in range(n)]
    if integer:
        scores = [rng.randint(-2, 5) for _ in range(n)]
    else:
        scores = [rng.uniform(0.1, 2.0) for _ in range(n)]
    bases = [rng.randint(0, cost_max) for _ in range(n)]
    unit = rng.choice([1, 2, 3, 8])
    lo = sum(min(c) for c in costs)
    hi = sum(max(c) for c in costs)
    budget = rng.randint(max(0, lo - 5), hi + 5)
    return costs, scores, bases, budget, unit


# ------------------------------------------------------------ oracle pins
def test_oracle_matches_exhaustive_enumeration():
    """Every selection enumerated on tiny problems (exact integer sums): the
    recurrence reaches the best objective, with a selection that fits."""
    rng = random.Random(0)
    for _ in range(400):
        costs, scores, bases, budget, unit = random_problem(rng)
        best, optimal = ref.brute_force(costs, scores, bases, budget, unit)
        got = ref.select(costs, scores, bases, budget, unit)
        if best is None:
            assert got is None
            continue
        choices, obj = got
        assert obj == best
        assert choices in optimal
        wq, bq = ref.quantize(costs, budget, unit)
        assert sum(wq[i][j] for i, j in enumerate(choices)) <= bq


def test_oracle_closed_forms():
    # Ample budget, positive scores: every weight keeps its largest candidate.
    costs = [[8, 16, 24], [40, 48], [5]]
    got, _ = ref.select(costs, [1.0, 0.5, 2.0], [10, 44, 5], budget=10 ** 6, unit=1)
    assert got == [2, 1, 0]
    # Budget exactly the cheapest selection: only that one fits.
    got, obj = ref.select(costs, [1.0, 0.5, 2.0], [10, 44, 5], budget=8 + 40 + 5, unit=1)
    assert got == [0, 0, 0] and obj == 1.0 * (8 - 10) + 0.5 * (40 - 44) + 0.0
    # Room for one upgrade: it goes to the more important weight.
    got, _ = ref.select([[10, 20], [10, 20]], [1.0, 3.0], [15, 15], budget=30, unit=1)
    assert got == [0, 1]
    # Nothing fits.
    assert ref.select([[10, 20], [10, 20]], [1.0, 3.0], [15, 15], budget=19, unit=1) is None


def test_oracle_budget_guarantee():
    """Costs rounded up, budget down: the true parameter count of every
    selection stays within the budget (the guarantee GAC claims)."""
    rng = random.Random(1)
    for _ in range(300):
        costs, scores, bases, budget, unit = random_problem(rng, n_max=6, m_max=5, cost_max=200,
                                                            integer=False)
        got = ref.select(costs, scores, bases, budget, unit)
        if got is not None:
            assert sum(costs[i][j] for i, j in enumerate(got[0])) <= budget


def read_golden(name):
    out = {}
    for line in open(os.path.join(HERE, "golden", name)):
        line = line.split("#", 1)[0].split()
        if line:
            out[line[0]] = line[1]
    return out


def test_budget_quantization_example():
    """The section's example: 100 matrices of 1024×1024 at ρ = 15%."""
    g = read_golden("gac_budget_quantization.txt")
    n, rows, cols = int(g["matrices"]), int(g["rows"]), int(g["cols"])
    rho, align = float(g["rho"]), int(g["align"])
    budget = math.floor((1 - rho) * n * rows * cols)
    unit = align * rows  # u = 8·M_min
    assert unit == int(g["unit"])
    # Raw table ~1e8 entries, quantized ~1e4, a reduction of u ≈ 8000×.
    assert 0.5 < budget / float(g["raw_entries_approx"]) < 2
    _, bq = ref.quantize([[0]], budget, unit)
    assert bq == 10880  # ⌊0.85·100·1024² / 8192⌋
    assert 0.75 < bq / float(g["quantized_entries_approx"]) < 1.25
    assert abs(unit / float(g["reduction_approx"]) - 1) < 0.05


# ------------------------------------------------------------ product parity
def test_c_solver_matches_oracle_bit_for_bit(L):
    rng = random.Random(2)
    for k in range(300):
        costs, scores, bases, budget, unit = random_problem(
            rng, n_max=12, m_max=8, cost_max=5000, integer=(k % 3 == 0))
        want = ref.select(costs, scores, bases, budget, unit)
        if want is None:
            with pytest.raises(lr.LrError) as e:
                lr.gac_select(costs, scores, bases, budget, unit)
            assert e.value.code == lr.LR_ERR_INFEASIBLE
            continue
        choices, obj = lr.gac_select(costs, scores, bases, budget, unit)
        assert choices == want[0]
        assert obj == want[1]  # the same fp64 sums in the same order


def test_c_solver_matches_oracle_on_a_32_layer_plan(L):
    """Full size: 224 Llama-3-8B-shaped weights, quantized budget ≈ 1.4e5."""
    ws = [gac.Weight(**d) for d in lrgen.gac_model(32, seed=11)]
    p = gac.plan(ws)
    cands = [gac.candidates(w) for w in ws]
    costs = [[c for _, c in cs] for cs in cands]
    bases = [int(round(w.r_star * w.step_cost)) for w in ws]
    want, obj = ref.select(costs, [w.score for w in ws], bases, p.budget, p.unit)
    assert [p.ranks[w.name] for w in ws] == [cands[i][j][0] for i, j in enumerate(want)]
    assert p.objective == obj
    assert p.total_params <= p.budget
    assert p.aligned_fraction == 1.0


def test_c_solver_argument_errors(L):
    i, q, d = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    n_cand = (i * 1)(2)
    cost = (q * 2)(10, 20)
    score = (d * 1)(1.0)
    base = (q * 1)(15)
    choice = (i * 1)(-7)
    ok = L.lr_gac_select(1, n_cand, cost, score, base, 40, 1, choice, None)
    assert ok == lr.LR_OK and choice[0] == 1
    E = lr.LR_ERR_INVALID_ARG
    assert L.lr_gac_select(0, n_cand, cost, score, base, 40, 1, choice, None) == E
    assert L.lr_gac_select(1, None, cost, score, base, 40, 1, choice, None) == E
    assert L.lr_gac_select(1, n_cand, cost, score, base, -1, 1, choice, None) == E
    assert L.lr_gac_select(1, n_cand, cost, score, base, 40, 0, choice, None) == E
    assert L.lr_gac_select(1, (i * 1)(0), cost, score, base, 40, 1, choice, None) == E
    assert L.lr_gac_select(1, (i * 1)(256), cost, score, base, 40, 1, choice, None) == E
    assert L.lr_gac_select(1, n_cand, (q * 2)(-1, 20), score, base, 40, 1, choice, None) == E
    assert L.lr_gac_select(1, n_cand, cost, (d * 1)(float("nan")), base, 40, 1, choice,
                           None) == E
    # Infeasible leaves choice untouched; an oversized table is refused.
    choice[0] = -7
    assert L.lr_gac_select(1, n_cand, cost, score, base, 9, 1, choice, None) == \
        lr.LR_ERR_INFEASIBLE
    assert choice[0] == -7
    assert L.lr_gac_select(1, n_cand, cost, score, base, 1 << 40, 1, choice, None) == \
        lr.LR_ERR_UNSUPPORTED
    assert lr.status_string(lr.LR_ERR_INFEASIBLE) == "LR_ERR_INFEASIBLE"


# ------------------------------------------------------------ host logic
def test_sweep_ranks_reproduces_the_sections_example():
    """§4.2: d* = 107.3 gives the candidate set {96, 104, 112, 128}."""
    assert gac.sweep_ranks(107.3) == [96, 104, 112, 128]
    assert gac.sweep_ranks(2.0) == [8, 32]
    assert gac.sweep_ranks(1741.0, limit=4096) == [1736, 1744, 1752, 1760]
    assert all(d % 8 == 0 for d in gac.sweep_ranks(3000.5))
    with pytest.raises(ValueError):
        gac.sweep_ranks(0.0)


def test_drop_cliffs():
    ranks = [96, 104, 112, 128]
    # Smooth: time grows with rank, nothing dropped.
    assert gac.drop_cliffs(ranks, {96: 1.0, 104: 1.05, 112: 1.1, 128: 1.2}) == ranks
    # 104 is slower than 128 by more than 5%: a cliff.
    assert gac.drop_cliffs(ranks, {96: 1.0, 104: 1.4, 112: 1.1, 128: 1.2}) == [96, 112, 128]
    # Within the tolerance: kept.
    assert gac.drop_cliffs(ranks, {96: 1.0, 104: 1.12, 112: 1.1, 128: 1.2}) == ranks
    # Unmeasured ranks are kept.
    assert gac.drop_cliffs(ranks, {96: 2.0, 128: 1.0}) == [104, 112, 128]


def test_candidates_and_dense_fallback():
    # q (4096×4096): break-even rank 2048.  r* = 1000 stays factorised.
    w = gac.Weight("q", 4096, 4096, 1000.0)
    c = gac.candidates(w)
    assert [r for r, _ in c] == [992, 1000, 1008, 1024]
    assert all(p == r * 8192 for r, p in c)
    # r* = 2045: ranks at or past 2048 become one dense candidate.
    c = gac.candidates(gac.Weight("q", 4096, 4096, 2045.0))
    assert [r for r, _ in c] == [2040, gac.DENSE]
    assert c[-1][1] == 4096 * 4096
    # Far past the break-even: dense only.
    c = gac.candidates(gac.Weight("q", 4096, 4096, 3000.0))
    assert c == [(gac.DENSE, 4096 * 4096)]


def test_plan_keeps_the_budget_and_aligns_every_rank(L):
    ws = [gac.Weight(**d) for d in lrgen.gac_model(2, seed=3)]
    p = gac.plan(ws)
    assert p.budget == gac.budget_for(ws)
    assert p.total_params <= p.budget
    assert p.aligned_fraction == 1.0
    assert p.unit == 8 * (4096 + 1024)
    for w in ws:
        r = p.ranks[w.name]
        assert r is gac.DENSE or (r % 8 == 0 and r * w.step_cost < w.dense_cost)
    # Measured times that make one swept rank a cliff keep it out.
    w0 = ws[0]
    ranks = gac.sweep_ranks(w0.r_star, limit=min(w0.K, w0.N))
    times = {w0.name: {d: 1.0 + 0.001 * d for d in ranks}}
    times[w0.name][ranks[0]] = 10.0
    p2 = gac.plan(ws, times=times)
    assert p2.ranks[w0.name] != ranks[0]
    # A budget below the cheapest selection is infeasible.
    with pytest.raises(lr.LrError) as e:
        gac.plan(ws, budget=1000)
    assert e.value.code == lr.LR_ERR_INFEASIBLE


def test_sweep_plan_and_times_by_weight():
    ws = [gac.Weight("a", 4096, 4096, 1000.0), gac.Weight("b", 4096, 4096, 1010.0),
          gac.Weight("c", 4096, 1024, 300.0)]
    sp = gac.sweep_plan(ws)
    assert set(sp) == {(4096, 4096), (4096, 1024)}
    assert sp[(4096, 4096)] == sorted(set(gac.sweep_ranks(1000.0, limit=4096))
                                      | set(gac.sweep_ranks(1010.0, limit=4096)))
    assert sp[(4096, 1024)] == gac.sweep_ranks(300.0, limit=1024)
    shape_times = {"4096x4096": {str(r): 1.0 + r * 1e-3 for r in sp[(4096, 4096)]}}
    wt = gac.times_by_weight(ws, shape_times)
    assert set(wt) == {"a", "b"}  # no timings for the 4096x1024 shape
    assert wt["a"][1000] == pytest.approx(2.0)
    assert gac.times_by_weight(ws, {(4096, 1024): {304: 3.0}}) == {"c": {304: 3.0}}


def test_c_solver_largest_candidate_index(L):
    """255 candidates (the most a weight may have): the last index is
    reachable and the result still equals the oracle's."""
    costs = [list(range(0, 255 * 3, 3)), [5, 9]]
    scores, bases = [1.0, 2.0], [100, 7]
    for budget in (10 ** 6, 400, 9):
        want = ref.select(costs, scores, bases, budget, 1)
        got = lr.gac_select(costs, scores, bases, budget, 1)
        assert got[0] == want[0] and got[1] == want[1]
    assert lr.gac_select(costs, scores, bases, 10 ** 6, 1)[0] == [254, 1]


def test_plan_with_the_measured_b200_sweep():
    """The committed B200 dimension sweep (`bench.py --gac-sweep`, M = 2048,
    every rank the 32-layer plan may choose for its four weight shapes) as
    the planner's cliff filter: the documented outcome (140 candidate ranks
    dropped, every chosen rank a multiple of 8, the plan's objective
    unchanged by the filter) holds on the stored data."""
    import json
    import os
    from rank_linear_layers_b200 import gac
    import lrgen
    path = os.path.join(os.path.dirname(gac.__file__), "gac_sweep_b200.json")
    with open(path) as f:
        sweep = json.load(f)
    assert sweep["M"] == 2048 and sweep["status"] == 0
    ws = [gac.Weight(**d) for d in lrgen.gac_model(32, 11)]
    wt = gac.times_by_weight(ws, sweep["times_us"])
    cliffs = 0
    for w in ws:
        swept = gac.sweep_ranks(w.r_star, limit=min(w.K, w.N))
        cliffs += len(swept) - len(gac.drop_cliffs(swept, wt.get(w.name, {}), 0.05))
    assert cliffs == 140
    measured = gac.plan(ws, times=wt)
    plain = gac.plan(ws)
    assert measured.aligned_fraction == 1.0
    assert measured.objective == plain.objective

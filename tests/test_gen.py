"""Pins for the seeded input generator (no GPU)."""
from fractions import Fraction
import math

import numpy as np
import pytest

import lrgen


def test_splitmix64_reference_stream():
    # The first outputs of the SplitMix64 reference stream started at state
    # 1234567 (state += 0x9E3779B97F4A7C15, then the finaliser).
    z = np.uint64(1234567) + (np.arange(5, dtype=np.uint64) + np.uint64(1)) * lrgen.GAMMA
    got = [int(v) for v in lrgen.splitmix64(z)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]


def _bf16_nearest_even_exact(x: float) -> float:
    """bf16 nearest-even by exact rational search (independent of frexp/rint)."""
    if x == 0.0:
        return 0.0
    fx = Fraction(x)
    e = math.floor(math.log2(abs(x)))
    while Fraction(2) ** e > abs(fx):
        e -= 1
    while Fraction(2) ** (e + 1) <= abs(fx):
        e += 1
    ulp = Fraction(2) ** (e - 7)
    q = abs(fx) / ulp
    lo = math.floor(q)
    rem = q - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    v = lo * ulp
    return float(v if x > 0 else -v)


def test_bf16_rounding_is_nearest_even():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-6, 6, 3000),
                        # exact ties between two bf16 neighbours
                        (np.arange(256, 512) + 0.5) * 2.0 ** -8,
                        -(np.arange(256, 512) + 0.5) * 2.0 ** -3])
    got = lrgen.bf16_to_f64(lrgen.bf16_bits(x))
    want = np.array([_bf16_nearest_even_exact(float(v)) for v in x])
    assert np.array_equal(got, want)


def test_bf16_roundtrip_of_representable_values():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    v = lrgen.bf16_to_f64(bits)
    ok = np.isfinite(v) & ((np.abs(v) >= 2.0 ** -120) | (v == 0)) & (np.abs(v) < 2.0 ** 127)
    back = lrgen.bf16_bits(v[ok])
    assert np.array_equal(back, bits[ok])


def test_normal_moments_and_determinism():
    x = lrgen.normal(0, 1, 1 << 18)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    assert np.array_equal(x[1000:2000], lrgen.normal(0, 1, 1000, start=1000))
    assert not np.array_equal(lrgen.normal(0, 1, 100), lrgen.normal(0, 2, 100))
    assert not np.array_equal(lrgen.normal(0, 1, 100), lrgen.normal(1, 1, 100))


def test_fan_in_scaling():
    p = lrgen.lowrank_problem(8, 4096, 300, 1024, seed=0)
    A = lrgen.bf16_to_f64(p["A"])
    B = lrgen.bf16_to_f64(p["B"])
    assert abs(A.std() * math.sqrt(4096) - 1) < 0.02
    assert abs(B.std() * math.sqrt(300) - 1) < 0.02


def test_layer_ranks_within_bounds_and_unaligned_allowed():
    for n_int in (14336, 12203):
        ranks = lrgen.layer_ranks(7, n_int)
        for name, K, N, _ in lrgen.LAYER_PROJECTIONS:
            if name in ("gate", "up"):
                N = n_int
            if name == "down":
                K = n_int
            m = min(K, N)
            assert math.ceil(0.35 * m) <= ranks[name] <= math.floor(0.85 * m)
    assert any(r % 8 for r in lrgen.layer_ranks(7).values())


@pytest.mark.slow
def test_prefill_svd_construction_eckart_young():
    # A = U_r·Σ_r, B = V_rᵀ with σ_i = i^-0.5, i = 1..4096, r = 1741.
    # ‖A·B‖_F² = Σ_{i<=r} 1/i and ‖W − A·B‖_F² = Σ_{i>r} 1/i for W = U·Σ·Vᵀ.
    K = N = 4096
    r = 1741
    p = lrgen.svd_problem(M=4, K=K, N=N, r=r, seed=0, keep_f64=True)
    U, V, A64, B64, s = p["U"], p["V"], p["A64"], p["B64"], p["sigma"]
    assert np.abs(U.T @ U - np.eye(K)).max() < 1e-12
    assert np.abs(V.T @ V - np.eye(N)).max() < 1e-12
    AB = A64 @ B64
    head = sum(1.0 / i for i in range(1, r + 1))
    tail = sum(1.0 / i for i in range(r + 1, K + 1))
    assert abs(np.sum(AB * AB) - head) < 1e-9
    assert abs(head - 8.03972) < 1e-5 and abs(tail - 0.85539) < 1e-5
    W = (U * s[None, :]) @ V.T
    R = W - AB
    assert abs(np.sum(R * R) - tail) < 1e-9
    # The bf16 factors are the fp64 products rounded once.
    assert np.array_equal(p["A"], lrgen.bf16_bits(A64))
    assert np.array_equal(p["B"], lrgen.bf16_bits(B64))
    # Statistical sanity of the workload: for X ~ N(0,1) a row of X·A·B has
    # expected squared norm Σ_{i<=r} σ_i² (U and V orthogonal), so
    # RMS(Y) = sqrt(Σ_{i<=r} (1/i) / N) ≈ 0.0443.  64 rows: the estimate's
    # standard deviation is about 1.4%.
    import oracle
    X = lrgen.normal_bf16(0, 77, (64, K), 1.0)
    Y = oracle.lr_linear(X, p["A"], p["B"])
    expect = math.sqrt(head / N)
    assert abs(expect - 0.0443) < 1e-4
    assert abs(float(np.sqrt(np.mean(Y ** 2))) / expect - 1) < 0.06


def test_row_blocks_are_rows_of_the_whole():
    """normal_bf16(..., row0=k): rows k .. k + rows - 1 of the matrix drawn
    whole (counter-based: any row block can be drawn on its own)."""
    import numpy as np
    import lrgen
    whole = lrgen.normal_bf16(3, 7, (11, 13), 0.5)
    parts = [lrgen.normal_bf16(3, 7, (n, 13), 0.5, row0=k) for k, n in [(0, 4), (4, 1), (5, 6)]]
    assert np.array_equal(np.concatenate(parts), whole)
    assert not np.array_equal(lrgen.normal_bf16(3, 7, (4, 13), 0.5, row0=1), whole[:4])

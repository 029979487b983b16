"""Host-side accounting pinned to the pages' worked example (no GPU)."""
import os

from rank_linear_layers_b200 import accounting as acc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "keep_ratio_example.txt")


def _golden():
    layers, vals = [], {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *rest = line.split()
        if key == "layer":
            layers.append(tuple(int(v) for v in rest))
        else:
            vals[key] = rest
    return layers, vals


def test_keep_ratio_worked_example():
    layers, vals = _golden()
    num, den = acc.keep_ratio_terms(layers)
    assert num == int(vals["numerator"][0])
    assert den == int(vals["denominator"][0])
    assert round(acc.keep_ratio(layers), 3) == float(vals["ratio_3dp"][0])
    fr = [k / min(m, n) for m, n, k in layers]
    assert fr == [float(v) for v in vals["rank_fraction"]]


def test_keep_ratio_is_sum_then_divide():
    # Not the mean of per-layer ratios.
    layers = [(4096, 4096, 1024), (4096, 11008, 2048)]
    mean_of_ratios = sum(k * (m + n) / (m * n) for m, n, k in layers) / 2
    assert abs(acc.keep_ratio(layers) - mean_of_ratios) > 0.01


def test_prefill_q_proj_keep_ratio():
    # r = 1741 of 4096×4096 keeps 1741·8192/4096² ≈ 0.850: ρ = 15% fewer parameters.
    assert abs(acc.keep_ratio([(4096, 4096, 1741)]) - 0.8501) < 1e-4


def test_work_formulas():
    assert acc.flops(2048, 4096, 1741, 4096) == 2 * 2048 * 1741 * 8192
    assert acc.algorithmic_bytes(16, 256, 107, 256) == (16 * 256 + 256 * 107 + 107 * 256 + 16 * 256) * 2
    assert abs(acc.break_even_rank(4096, 1024) - 819.2) < 1e-9
    rf = acc.roofline(acc.flops(2048, 4096, 1741, 4096), acc.algorithmic_bytes(2048, 4096, 1741, 4096),
                      2250.0, 8000.0)
    assert rf.bound == "tensor" and abs(rf.t_roof_s * 1e6 - 26.0) < 0.1


def test_group_counts_shared_input_once():
    projs = [dict(K=4096, r=100, N=4096, x="a"), dict(K=4096, r=50, N=1024, x="a")]
    fl, by = acc.group_work(8, projs)
    assert fl == acc.flops(8, 4096, 100, 4096) + acc.flops(8, 4096, 50, 1024)
    assert by == acc.algorithmic_bytes(8, 4096, 100, 4096) + acc.algorithmic_bytes(8, 4096, 50, 1024) - 8 * 4096 * 2

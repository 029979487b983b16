"""The gated output of lr_linear_group (lr_proj.silu_gate): the up
projection's Y is silu(G) · P, G the gate projection's stored output and P
the up projection's own fp32 product.  Paths: fused into the streamed
decode launch (M <= 8); an fp32 area plus one elementwise launch after the
two-launch decode kernels (M = 12) and after the prefill group launch
(M = 300).

* fp32 gate and fp32 up output: against the fp64 oracle, SiLU and the
  product applied on the CPU to the oracle's outputs, at the parity bar.
* bf16 gate: the product uses the gate as stored: it equals silu(G) · P,
  G the run's own stored gate and P the up output of the same group run
  without the gate link, up to fp32 rounding (1e-4·RMS; the gate's own
  rounding to bf16 would show as about 1e-3·RMS).
* bf16 up output: within one bf16 ulp (plus 1e-5·RMS near zero) of the
  fp32 output rounded (two launches may add partial sums in another
  order).
"""
import numpy as np
import pytest

import lrgen
import oracle
from helpers import compare, rn_bf16, to_dev, to_f64

pytestmark = pytest.mark.gpu

K, N = 4096, 2000


def silu(x):
    return x / (1.0 + np.exp(-x))


def _problems(M, seed=5):
    pg = lrgen.lowrank_problem(M, K, 1505, N, seed=seed, bias=False)
    pu = lrgen.lowrank_problem(M, K, 2125, N, seed=seed + 1, bias=True, tid_base=20)
    pu["X"] = pg["X"]
    po = lrgen.lowrank_problem(M, 2000, 300, 512, seed=seed + 2, bias=False, tid_base=40)
    return pg, pu, po


def _run(M, gate_f32, up_f32, link=True, seed=5):
    """Group (up gated by gate, plus an unrelated projection); returns the
    host copies of up, gate and other outputs and the launch count."""
    import torch
    import rank_linear_layers_b200 as lr
    pg, pu, po = _problems(M, seed)
    X = to_dev(pg["X"])
    G = torch.full((M, N), float("nan"), dtype=torch.float32 if gate_f32 else torch.bfloat16,
                   device="cuda")
    U = torch.full((M, N), float("nan"), dtype=torch.float32 if up_f32 else torch.bfloat16,
                   device="cuda")
    O = torch.full((M, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    entries = [dict(X=X, A=to_dev(pu["A"]), B=to_dev(pu["B"]), bias=to_dev(pu["bias"]), Y=U,
                    silu_gate=2 if link else None),
               dict(X=to_dev(po["X"]), A=to_dev(po["A"]), B=to_dev(po["B"]), Y=O),
               dict(X=X, A=to_dev(pg["A"]), B=to_dev(pg["B"]), Y=G)]
    n0 = lr.kernel_launch_count()
    lr.lr_linear_group(entries, M)
    launches = lr.kernel_launch_count() - n0
    torch.cuda.synchronize()
    assert lr.last_device_status() == lr.LR_OK
    host = lambda t: t.double().cpu().numpy() if t.dtype == torch.float32 else to_f64(t)
    return host(U), host(G), host(O), launches


@pytest.mark.parametrize("M", [1, 4, 12, 300])
def test_silu_gate_against_oracle(M):
    pg, pu, po = _problems(M)
    Yu, Yg, Yo, launches = _run(M, gate_f32=True, up_f32=True)
    gref = oracle.lr_linear(pg["X"], pg["A"], pg["B"], None)
    uref = oracle.lr_linear(pu["X"], pu["A"], pu["B"], pu["bias"])
    compare(Yu, silu(gref) * uref, f"silu(gate)·up M={M}")
    compare(Yg, gref, f"gate M={M}")
    compare(Yo, oracle.lr_linear(po["X"], po["A"], po["B"], None), f"other projection M={M}")
    if M <= 8:
        assert launches == 1  # formed inside the streamed launch


@pytest.mark.parametrize("M", [1, 12, 300])
def test_silu_gate_uses_the_stored_bf16_gate(M):
    Yu, Yg, _, _ = _run(M, gate_f32=False, up_f32=True)
    P, _, _, _ = _run(M, gate_f32=False, up_f32=True, link=False)
    want = silu(Yg) * P
    rms = np.sqrt(np.mean(want ** 2))
    assert np.max(np.abs(Yu - want)) <= 1e-4 * rms, \
        f"M={M}: gated output is not silu(stored gate) · product"


@pytest.mark.parametrize("M", [1, 300])
def test_silu_gate_bf16_output_is_the_fp32_one_rounded(M):
    Y32, _, _, _ = _run(M, gate_f32=True, up_f32=True)
    Y16, _, _, _ = _run(M, gate_f32=True, up_f32=False)
    r = rn_bf16(Y32.astype(np.float32))
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(r), 1e-30))) - 7)
    # Near zero the two launches' fp32 sums differ by more than a bf16 ulp
    # of the value itself: allow that run-to-run noise (1e-5·RMS) too.
    noise = 1e-5 * np.sqrt(np.mean(r ** 2))
    assert np.all(np.abs(Y16 - r) <= ulp + noise), f"M={M}: bf16 output off the rounded fp32 one"

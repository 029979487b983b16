"""Benchmark of the low-rank linear layer Y = (X·A)·B on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one step = one lr_linear call over one batch): the prefill q_proj
shape of Llama-3-8B, X [2048, 4096] ~ N(0,1), A = U·Σ [4096, 1741],
B = Vᵀ [1741, 4096], U and V Haar orthogonal, σ_i = i^-0.5 (bf16 inputs,
fp32 accumulation).  Rank 1741 is not a multiple of 8: keeping 15% fewer
parameters than the 4096×4096 layer, as in the GAC paper's ASVD setting.

Prints one JSON line (rank 0).  `value` is whole-job TFLOP/s (2·M·r·(K+N)
FLOPs per step per rank, summed over ranks, over the max-over-ranks device
time).  Inputs rotate over enough copies to exceed twice the L2 size, so no
step reads its operands from L2.  Also reported: the roofline fraction of the
prefill kernels, the end-to-end rate through the host-buffer C ABI call, the
decode (M = 1, 4, 16) bandwidth of the Llama-3-8B MLP shapes, the time per
call of the small single layer (16×256 · 256×107), the fp64 CPU
oracle timed on a bounded sample (the CPU baseline), SM clocks sampled during
the timed region and the number of library kernels launched.

With --gpus N > 1 (torchrun), every rank runs its own batch with the same
factors (rows of X are independent): weak scaling, no data-path collective.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import lrgen  # noqa: E402
from rank_linear_layers_b200 import accounting as acc  # noqa: E402

M, K, R, N = 2048, 4096, 1741, 4096
WORKLOAD = "prefill q_proj: X[2048,4096] · A[4096,1741] (U·Σ, σ_i=i^-0.5) · B[1741,4096] (Vᵀ), bf16"
CACHE = os.environ.get("LR_BENCH_CACHE", "/tmp/lr_bench_inputs")
DECODE_SHAPES = [("gate_up", 4096, 2867, 14336), ("down", 14336, 2867, 4096)]


# B200 nominal figures (dense bf16 tensor throughput, HBM3e bandwidth of the
# HGX part): the denominators of `frac_spec`.  The targets (70% prefill, 80%
# decode) are stated against the measured peaks (`frac`); `frac_spec` is reported
# beside them.
SPEC_PEAKS = {"bf16_tflops": 2250.0, "hbm_gbs": 7700.0,
              "source": "B200 nominal: 2.25 PFLOP/s dense bf16, 7.7 TB/s HBM3e"}


def fallback_peaks():
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    except Exception:
        return fallback_peaks()


# Device sources of the kernels the prefill step launches (the chain GEMM and
# the repack); an ncu summary's traffic figure is used only while they are
# unchanged.
PREFILL_SOURCES = ("lr_internal.h", "lr_load.cuh", "lr_ptx.cuh", "lr_repack.cu", "lr_umma.cu")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rank_linear_layers_b200", "csrc")
    for fn in PREFILL_SOURCES:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", name)
    try:
        vals = {}
        for line in open(path):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
        if vals.get("kernel_source_hash") != kernel_source_hash():
            return None
        return float(vals["dram_bytes_per_step"])
    except Exception:
        return None


def prefill_inputs():
    """The prefill problem (cached on disk: the QR of two 4096² matrices takes a while)."""
    os.makedirs(CACHE, exist_ok=True)
    f = os.path.join(CACHE, f"q_proj_{M}_{K}_{R}_{N}_seed0.npz")
    if os.path.exists(f):
        z = np.load(f)
        return {"X": z["X"], "A": z["A"], "B": z["B"], "bias": None}
    p = lrgen.svd_problem(M=M, K=K, N=N, r=R, seed=0)
    try:
        np.savez(f + ".tmp.npz", X=p["X"], A=p["A"], B=p["B"])
        os.replace(f + ".tmp.npz", f)
    except OSError:
        pass
    return p


def rank_rows(rank, rows=None):
    """Rank `rank`'s rows of the whole job's batch of X: rows rank·M ..
    rank·M + M - 1 of one matrix drawn by the prefill generator (X ~ N(0,1),
    seed 0), the factors replicated on every rank (data parallel, weak
    scaling: no data-path collective).  `rows` overrides M (tests)."""
    m = M if rows is None else rows
    return lrgen.normal_bf16(0, lrgen.TENSOR_ID["X"], (m, K), 1.0, row0=rank * m)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled every 5 ms through NVML
    while the timed region runs (read-only queries)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.reasons = set()
        self._stop = None
        self._thread = None
        self.max_mhz = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            dev = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            idx = int(dev.split(",")[self.index]) if dev and dev.split(",")[0].isdigit() else self.index
            h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                    mask = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                    for name, bit in self.REASONS.items():
                        if mask & bit:
                            self.reasons.add(name)
                except Exception:
                    pass
                self._stop.wait(0.005)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return None
        self._stop.set()
        self._thread.join(timeout=2)
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": sorted(self.reasons)}


# ---------------------------------------------------------------- timing
def time_steps(fn, steps, warmup, flush=None):
    """Device time of `steps` calls (CUDA events on the launching stream)."""
    import torch
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for i in range(steps):
        fn(warmup + i)
    e1.record(s)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e-3


def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce(x, world, op):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x, world):
    """Timing across ranks: the slowest rank's device time."""
    import torch.distributed as dist
    return x if world == 1 else _reduce(x, world, dist.ReduceOp.MAX)


def sum_over_ranks(x, world):
    """Work across ranks: every rank's units count."""
    import torch.distributed as dist
    return x if world == 1 else _reduce(x, world, dist.ReduceOp.SUM)


def aggregate(flops_per_rank, seconds_per_rank, world):
    """Whole-job TFLOP/s: units of all ranks over the max-over-ranks time."""
    t = max_over_ranks(seconds_per_rank, world)
    return sum_over_ranks(flops_per_rank, world) / t / 1e12, t


# ---------------------------------------------------------------- CPU baseline
def cpu_baseline(p, check=None, budget_s=12.0):
    """The fp64 oracle on a bounded row sample of the same workload.  Its
    first chunk is `check` = (rows, the GPU's bf16 output of those rows as
    fp64), whose parity with the oracle is returned beside the timing."""
    import oracle
    threads = oracle.default_threads()
    rows_per_chunk = 32
    done = 0
    parity = None
    t0 = time.perf_counter()
    if check is not None:
        rows, Yg = check
        Yr = oracle.lr_linear(p["X"], p["A"], p["B"], None, rows=rows, threads=threads)
        done += len(rows)
        rms = float(np.sqrt(np.mean(Yr ** 2)))
        parity = {"rows": int(len(rows)), "max_err_over_rms": float(np.abs(Yg - Yr).max() / rms),
                  "rel_fro": float(np.linalg.norm(Yg - Yr) / np.linalg.norm(Yr))}
    rng = np.random.default_rng(1)
    while time.perf_counter() - t0 < budget_s and done < 4 * M:
        rows = rng.choice(M, rows_per_chunk, replace=False)
        oracle.lr_linear(p["X"], p["A"], p["B"], None, rows=rows, threads=threads)
        done += rows_per_chunk
    dt = time.perf_counter() - t0
    fl = acc.flops(done, K, R, N)
    cb = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
          "sample": f"{done} rows of X (of {M}) through the fp64 oracle, {dt:.1f} s"}
    return cb, parity


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    p = prefill_inputs()
    # Each step is one bounded sample; time K of them after W warm-ups.
    import oracle
    threads = oracle.default_threads()
    rows_per_step = 64
    rng = np.random.default_rng(2)
    for _ in range(args.warmup):
        oracle.lr_linear(p["X"], p["A"], p["B"], None, rows=rng.choice(M, rows_per_step, replace=False),
                         threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.lr_linear(p["X"], p["A"], p["B"], None, rows=rng.choice(M, rows_per_step, replace=False),
                         threads=threads)
    dt = time.perf_counter() - t0
    value = acc.flops(rows_per_step * args.steps, K, R, N) / dt / 1e12
    cb = {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
          "sample": f"{rows_per_step} rows of X per step (of {M}), fp64 oracle"}
    line = {
        "impl": "reference", "metric": metric_name(), "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / max(1, args.steps) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(), "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def _dev_bits(bits, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def sweep_times(lr, dev, l2, ranks, steps=20, warmup=3):
    """Time per call at M = K = N = 4096 for each rank.  X ~ N(0,1),
    A ~ N(0, 1/K), B ~ N(0, 1/1000): the A and B of each rank are the leading
    columns / rows of one seeded draw (values do not affect the timing)."""
    import torch
    Mw, Kw, Nw = 4096, 4096, 4096
    rmax = max(ranks)
    X0 = _dev_bits(lrgen.normal_bf16(0, 1, (Mw, Kw)), dev)
    Af = _dev_bits(lrgen.normal_bf16(0, 2, (Kw, rmax), 1.0 / math.sqrt(Kw)), dev)
    Bf = _dev_bits(lrgen.normal_bf16(0, 3, (rmax, Nw), 1.0 / math.sqrt(1000)), dev)
    Xs = [X0] + [X0.clone() for _ in range(max(1, math.ceil(2 * l2 / (X0.numel() * 2))))]
    Y = torch.empty((Mw, Nw), dtype=torch.bfloat16, device=dev)
    out = {}
    for r in ranks:
        A = Af[:, :r].contiguous()
        B = Bf[:r].contiguous()

        def st(i, A=A, B=B):
            lr.lr_linear(Xs[i % len(Xs)], A, B, None, Y=Y)
        tt = time_steps(st, steps, warmup) / steps
        out[r] = {"us": tt * 1e6, "ps_per_flop": tt / acc.flops(Mw, Kw, r, Nw) * 1e12}
    return out


def single_layer_bench(lr, dev, steps=200, warmup=20):
    """The small single layer, X [16,256] · A [256,107] · B [107,256] (seed 0,
    no bias): launch- and latency-bound, so its absolute time per call is
    the figure of merit.  Back-to-back calls on one stream, CUDA events."""
    try:
        import torch
        q = lrgen.lowrank_problem(16, 256, 107, 256, seed=0)
        X, A, B = (_dev_bits(q[k], dev) for k in ("X", "A", "B"))
        Y = torch.empty((16, 256), dtype=torch.bfloat16, device=dev)
        n0 = lr.kernel_launch_count()
        lr.lr_linear(X, A, B, None, Y=Y)
        per_call = lr.kernel_launch_count() - n0

        def st(i):
            lr.lr_linear(X, A, B, None, Y=Y)
        t = time_steps(st, steps, warmup) / steps
        out = {"us_per_call": t * 1e6, "gpu_launches_per_call": int(per_call),
               "flops": acc.flops(16, 256, 107, 256),
               "note": "M=16 K=256 r=107 N=256, one-CTA path, back-to-back calls"}
    except Exception as ex:  # pragma: no cover - reported, not hidden
        return {"error": str(ex)[:200]}
    # The launch floor: the same calls captured in one CUDA graph.  The
    # library keeps a workspace per stream, so the capture stream is warmed
    # up first (nothing is allocated while capturing).
    try:
        cs = torch.cuda.Stream(device=dev)
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cs):
            for i in range(3):
                st(i)
        cs.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cs):
            for i in range(steps):
                st(i)
        g.replay()
        torch.cuda.synchronize()
        cur = torch.cuda.current_stream()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        for _ in range(3):
            g.replay()
        e1.record(cur)
        torch.cuda.synchronize()
        out["graph_us_per_call"] = e0.elapsed_time(e1) * 1e3 / (3 * steps)
        del g
    except Exception as ex:  # pragma: no cover - reported, not hidden
        out["graph_error"] = str(ex)[:200]
    return out


MISALIGN_RANKS = list(range(1000, 1105)) + [64, 128, 512, 2048]


def misalignment_check(lr, dev, l2, ranks=MISALIGN_RANKS):
    """The misalignment sweep, M = K = N = 4096 at every r from 1000 to 1100
    (and the multiples of 8 around them) plus r = 64, 128, 512, 2048: each
    misaligned rank against the nearest multiple of 8 (both neighbours at
    r = 4 mod 8), in time per FLOP; and each rank's fraction of its roofline."""
    t = sweep_times(lr, dev, l2, list(ranks))
    worst, worst_r = 0.0, None
    rows = {}
    for r, v in t.items():
        if r % 8 == 0 or r < 1000 or r > 1100:
            continue
        lo, hi = r - r % 8, r - r % 8 + 8
        near = [lo] if r % 8 < 4 else ([hi] if r % 8 > 4 else [lo, hi])
        near = [n for n in near if n in t]
        if not near:
            continue
        dev_pct = max(v["ps_per_flop"] / t[n]["ps_per_flop"] - 1.0 for n in near)
        rows[r] = round(dev_pct * 100, 2)
        if dev_pct > worst:
            worst, worst_r = dev_pct, r
    peaks = load_peaks()
    frac = {}
    for r, v in t.items():
        roof = acc.roofline(acc.flops(4096, 4096, r, 4096), acc.algorithmic_bytes(4096, 4096, r, 4096),
                            peaks["bf16_tflops"], peaks["hbm_gbs"])
        frac[r] = round(roof.t_roof_s / (v["us"] * 1e-6), 3)
    return {"workload": "M=K=N=4096, r=1000..1100 step 1 and {64,128,512,2048}",
            "us": {r: round(v["us"], 2) for r, v in t.items()},
            "frac_roofline": frac,
            "pct_slower_than_nearest_aligned_per_flop": rows, "worst_pct": round(worst * 100, 2),
            "worst_rank": worst_r if worst > 0 else None, "target_pct": 5.0}


def layer_bench(lr, dev, peaks, n_int=14336):
    """A full factorised Llama-3-8B decoder layer through lr_linear_group."""
    import torch
    res = {}
    for Ml in (1, 4096):
        layer = lrgen.decoder_layer(Ml, seed=7, n_int=n_int)
        xs = {k: _dev_bits(v, dev) for k, v in layer["inputs"].items()}
        P = layer["projs"]
        packed = torch.empty((Ml, 2 * n_int), dtype=torch.bfloat16, device=dev)
        # At M = 1 the factors (~76 MB) would stay in L2 between steps: two
        # copies of them alternate.
        sets, keep = [], []
        Ys = {name: torch.empty((Ml, p["N"]), dtype=torch.bfloat16, device=dev)
              for name, p in P.items() if name not in ("gate", "up")}
        for copy in range(2 if Ml == 1 else 1):
            entries = []
            for name, p in P.items():
                A, B = _dev_bits(p["A"], dev), _dev_bits(p["B"], dev)
                keep += [A, B]
                e = dict(X=xs[p["x"]], A=A, B=B, K=p["K"], r=p["r"], N=p["N"])
                if name in ("gate", "up"):
                    e["Y_ptr"] = packed.data_ptr() + (0 if name == "gate" else 2 * n_int)
                    e["ld_y"] = 2 * n_int
                else:
                    e["Y"] = Ys[name]
                entries.append(e)
            sets.append(entries)
        step = lambda i: lr.lr_linear_group(sets[i % len(sets)], Ml)
        tl = time_steps(step, 20, 3) / 20
        projs = [dict(K=p["K"], r=p["r"], N=p["N"], x=p["x"]) for p in P.values()]
        fl, by = acc.group_work(Ml, projs)
        dense_by = sum(acc.dense_bytes(Ml, p["K"], p["N"]) for p in P.values())
        dense_fl = sum(acc.dense_flops(Ml, p["K"], p["N"]) for p in P.values())
        roof = acc.roofline(fl, by, peaks["bf16_tflops"], peaks["hbm_gbs"])
        droof = acc.roofline(dense_fl, dense_by, peaks["bf16_tflops"], peaks["hbm_gbs"])
        res[f"M{Ml}"] = {"us": tl * 1e6, "TFLOP/s": fl / tl / 1e12, "GB/s": by / tl / 1e9,
                         "roofline_us": roof.t_roof_s * 1e6, "frac_roofline": roof.t_roof_s / tl,
                         "dense_roofline_us": droof.t_roof_s * 1e6,
                         "ranks": layer["ranks"], "keep_ratio": acc.keep_ratio(
                             [(p["K"], p["N"], p["r"]) for p in P.values()])}
        if Ml == 1:
            # Back-to-back eager calls at M = 1 wait on the host (building the
            # call's table in Python); the same calls replayed from a CUDA
            # graph give the device time.
            tg = graph_us(step, 10, dev) * 1e-6
            res["M1"].update({"graph_us": tg * 1e6, "frac_roofline_graph": roof.t_roof_s / tg,
                              "launches_per_call": 1})
    return res


def graph_us(fn, calls, dev):
    """Device time per call of `calls` calls captured in one CUDA graph and
    replayed three times (the library keeps a workspace per stream, so the
    capture stream is warmed up first: nothing is allocated while capturing)."""
    import torch
    cs = torch.cuda.Stream(device=dev)
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs):
        for i in range(3):
            fn(i)
    cs.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cs):
        for i in range(calls):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for _ in range(3):
        g.replay()
    e1.record(cur)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / (3 * calls)


def metric_name():
    return "low-rank linear TFLOP/s (prefill) and GB/s (decode) as % of B200 roofline"


def config_dict():
    return {"workload": WORKLOAD, "M": M, "K": K, "r": R, "N": N, "r_mod_8": R % 8,
            "factors": "A=U·Σ, B=Vᵀ, Haar U,V, sigma_i=i^-0.5", "bias": False,
            "l2": "inputs rotate over copies totalling > 2x L2 between steps",
            "parallelism": "data-parallel rows of X, factors replicated (weak scaling)"}


# ---------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import rank_linear_layers_b200 as lr

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    p = prefill_inputs()

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    # This rank's rows of the whole job's batch (rank 0: the cached rows).
    X0 = to_dev(p["X"] if rank == 0 else rank_rows(rank))
    A0, B0 = to_dev(p["A"]), to_dev(p["B"])
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    step_bytes = (X0.numel() + A0.numel() + B0.numel()) * 2
    copies = max(2, math.ceil(2 * l2 / step_bytes) + 1)
    Xs = [X0] + [X0.clone() for _ in range(copies - 1)]
    As = [A0] + [A0.clone() for _ in range(copies - 1)]
    Bs = [B0] + [B0.clone() for _ in range(copies - 1)]
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

    def step(i):
        j = i % copies
        lr.lr_linear(Xs[j], As[j], Bs[j], None, Y=Y)

    # Correctness gate on the timed configuration: the device status now, and
    # 16 sampled output rows kept for the CPU-baseline leg, which checks them
    # against the oracle (rank 0, one GPU).
    step(0)
    torch.cuda.synchronize()
    if lr.last_device_status() != lr.LR_OK:
        raise RuntimeError("device status not OK")
    check_rows = np.random.default_rng(0).choice(M, 16, replace=False)
    check_Y = lrgen.bf16_to_f64(
        Y[torch.as_tensor(check_rows, device=dev)].cpu().view(torch.int16).numpy().view(np.uint16))

    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    launches0 = lr.kernel_launch_count()
    t = time_steps(step, args.steps, 0)
    launches_timed = lr.kernel_launch_count() - launches0
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    fl_step = acc.flops(M, K, R, N)
    value, t_max = aggregate(fl_step * args.steps, t, world)
    ms = t_max / args.steps * 1e3

    # Roofline of the prefill step: one launch of the tcgen05 chain kernel
    # (GEMM1 T = X·A and GEMM2 Y = T·B, all of the step's FLOPs), after one
    # repack launch for A (r = 1741 has 3482-byte rows).  `achieved` divides
    # the step's FLOPs by the step's time, so it includes the repack.
    peak = peaks.get("bf16_tflops") or fallback_peaks()["bf16_tflops"]
    achieved = fl_step / (t / args.steps) / 1e12
    traffic = recorded_traffic("chain_prefill_q_proj.txt")
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic,
                "frac_spec": achieved / SPEC_PEAKS["bf16_tflops"],
                "peak_spec": SPEC_PEAKS["bf16_tflops"], "peak_spec_source": SPEC_PEAKS["source"],
                "peak_kind": f"{peaks['source']} bf16 burst (cuBLAS 8192^3)",
                "kernel": "umma_chain_kernel (GEMM1 + GEMM2, one launch) + repack_rows_bulk_kernel (A) per step; achieved = step FLOPs / step time",
                "algorithmic_bytes_per_step": acc.algorithmic_bytes(M, K, R, N),
                "flops_per_step": fl_step}

    if args.profile:
        # Prefill steps only, for ncu captures of this command.
        if rank == 0:
            print(json.dumps({"profile_run": True, "ms_per_step": ms, "gpu_launches": int(launches_timed)}))
        return 0

    # Two more trials of the same K steps on this rank (the reported value is
    # the first): the spread of the per-step time across trials.
    trials = [t / args.steps * 1e3]
    try:
        for _ in range(2):
            trials.append(time_steps(step, args.steps, 0) / args.steps * 1e3)
    except Exception:  # pragma: no cover - the main figure stands alone
        pass

    # End to end through the host-buffer C ABI call (pinned host memory).
    e2e = None
    try:
        Xh = torch.from_numpy(p["X"].view(np.int16)).view(torch.bfloat16).pin_memory()
        Ah = torch.from_numpy(p["A"].view(np.int16)).view(torch.bfloat16).pin_memory()
        Bh = torch.from_numpy(p["B"].view(np.int16)).view(torch.bfloat16).pin_memory()
        Yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        e2e_steps = max(3, min(args.steps, 20))
        for _ in range(2):
            lr.lr_linear_host(Xh, Ah, Bh, None, Y=Yh)
        barrier(world)
        t0 = time.perf_counter()
        for _ in range(e2e_steps):
            lr.lr_linear_host(Xh, Ah, Bh, None, Y=Yh)
        te = max_over_ranks((time.perf_counter() - t0) / e2e_steps, world)
        e2e = {"value": sum_over_ranks(fl_step, world) / te / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int((Xh.numel() + Ah.numel() + Bh.numel()) * 2),
               "d2h_bytes_per_step": int(Yh.numel() * 2), "ms_per_step": te * 1e3,
               "steps": e2e_steps, "note": "lr_linear_host: X, A, B copied in and Y out every step"}
    except Exception as ex:  # pragma: no cover - reported, not hidden
        e2e = {"value": None, "unit": "TFLOP/s", "error": str(ex)[:200]}

    # Decode (M = 1, 4, 16) on the MLP shapes: bandwidth and % of HBM peak.
    decode = {}
    if not args.no_decode:
        for name, dk, dr, dn in DECODE_SHAPES:
            for dm in (1, 4, 16):
                q = lrgen.lowrank_problem(dm, dk, dr, dn, seed=0)
                Xd, Ad, Bd = to_dev(q["X"]), to_dev(q["A"]), to_dev(q["B"])
                cps = max(2, math.ceil(2 * l2 / ((Ad.numel() + Bd.numel()) * 2)) + 1)
                Ads = [Ad] + [Ad.clone() for _ in range(cps - 1)]
                Bds = [Bd] + [Bd.clone() for _ in range(cps - 1)]
                Yd = torch.empty((dm, dn), dtype=torch.bfloat16, device=dev)

                def dstep(i, Xd=Xd, Ads=Ads, Bds=Bds, Yd=Yd, cps=cps):
                    lr.lr_linear(Xd, Ads[i % cps], Bds[i % cps], None, Y=Yd)
                td = time_steps(dstep, 50, 5) / 50
                tg = graph_us(dstep, 2 * cps, dev) * 1e-6
                by = acc.algorithmic_bytes(dm, dk, dr, dn)
                decode[f"{name}_M{dm}"] = {
                    "us": td * 1e6, "GB/s": by / td / 1e9,
                    "frac_hbm": by / td / 1e9 / peaks["hbm_gbs"],
                    "frac_hbm_spec": by / td / 1e9 / SPEC_PEAKS["hbm_gbs"],
                    "graph_us": tg * 1e6, "frac_hbm_graph": by / tg / 1e9 / peaks["hbm_gbs"],
                    "dense_equiv_us_at_peak": acc.dense_bytes(dm, dk, dn) / (peaks["hbm_gbs"] * 1e9) * 1e6}
                del Ads, Bds

    # Dense X·W at the same M, K, N through the same kernels: is the
    # factorised layer (15% fewer parameters) still slower?
    dense = None
    if not args.no_extra:
        gen = torch.Generator(device=dev).manual_seed(0)
        Wd = [(torch.randn((K, N), generator=gen, device=dev) / math.sqrt(K)).to(torch.bfloat16)
              for _ in range(copies)]
        Yd = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

        def dstep(i):
            lr.lr_dense(Xs[i % copies], Wd[i % copies], None, Y=Yd)
        tdd = time_steps(dstep, args.steps, args.warmup) / args.steps
        dense = {"us": tdd * 1e6, "TFLOP/s": acc.dense_flops(M, K, N) / tdd / 1e12,
                 "lowrank_over_dense_time": (t / args.steps) / tdd,
                 "note": "lr_dense, same tcgen05 kernel, W [4096,4096] N(0,1/K)"}
        del Wd
    # The same prefill step with the factors stored once at an aligned pitch
    # (lr_factor_pitch: the "prepared weight" form, no per-call realignment
    # copy), and with an unrelated kernel between calls, so that nothing of
    # the previous call overlaps the next (no early copy either way).
    prepared = None
    if not args.no_extra:
        try:
            pa = lr.factor_pitch(R)
            Aps = []
            for j in range(copies):
                buf = torch.zeros((K, pa), dtype=torch.bfloat16, device=dev)
                buf[:, :R] = As[j]
                Aps.append(buf[:, :R])
            other = torch.empty(1 << 20, dtype=torch.float32, device=dev)

            def pstep(i):
                j = i % copies
                lr.lr_linear_strided(Xs[j], Aps[j], Bs[j], None, Y=Y)
            tp = time_steps(pstep, args.steps, args.warmup) / args.steps

            def istep(i):
                j = i % copies
                other.add_(1.0)
                lr.lr_linear(Xs[j], As[j], Bs[j], None, Y=Y)
            ti = time_steps(istep, args.steps, args.warmup) / args.steps

            def pistep(i):
                j = i % copies
                other.add_(1.0)
                lr.lr_linear_strided(Xs[j], Aps[j], Bs[j], None, Y=Y)
            tpi = time_steps(pistep, args.steps, args.warmup) / args.steps
            prepared = {
                "us": tp * 1e6, "TFLOP/s": fl_step / tp / 1e12, "frac": fl_step / tp / 1e12 / peak,
                "lda": pa,
                "interleaved_us": ti * 1e6, "prepared_interleaved_us": tpi * 1e6,
                "note": "A stored at pitch lr_factor_pitch(r) (no realignment copy); "
                        "interleaved: a 4 MB elementwise kernel between calls (its time included)"}
            del Aps
        except Exception as ex:  # pragma: no cover - reported, not hidden
            prepared = {"error": str(ex)[:200]}
    misalign = misalignment_check(lr, dev, l2) if not args.no_extra else None
    layer = layer_bench(lr, dev, peaks) if not args.no_extra else None
    layer_pruned = None
    if not args.no_extra:
        try:  # the pruned MLP (N_int = 12203: odd strides, 2-byte-aligned packed output)
            layer_pruned = layer_bench(lr, dev, peaks, n_int=12203)
        except Exception as ex:  # pragma: no cover - reported, not hidden
            layer_pruned = {"error": str(ex)[:200]}
    single = single_layer_bench(lr, dev) if not args.no_extra else None

    cb, parity = (cpu_baseline(p, check=(check_rows, check_Y)) if (rank == 0 and world == 1)
                  else (None, None))
    if rank == 0:
        line = {
            "metric": metric_name(), "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config_dict(), "roofline": roofline,
            "cpu_baseline": cb, "e2e": e2e, "gpu_launches": int(launches_timed),
            "clocks": clk, "parity": parity, "decode": decode, "dense": dense,
            "trials_ms_per_step": trials,
            "trial_spread_pct": (max(trials) - min(trials)) / statistics.median(trials) * 100,
            "misalignment": misalign, "prepared": prepared, "layer": layer,
            "layer_pruned": layer_pruned,
            "single_layer": single,
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the dense, misalignment and decoder-layer measurements")
    ap.add_argument("--sweep", action="store_true",
                    help="only the misalignment sweep r = 1000..1100 and {64,128,512,2048}")
    ap.add_argument("--profile", action="store_true",
                    help="only the timed prefill steps (for ncu captures); numbers are not a bench line")
    ap.add_argument("--gac-sweep", action="store_true",
                    help="only time lr_linear at the ranks the GAC planner sweeps, per weight shape")
    ap.add_argument("--gac-m", type=int, default=2048, help="tokens for --gac-sweep")
    ap.add_argument("--profile-layer", action="store_true",
                    help="only the decoder layer at M = 1 through lr_linear_group (for ncu captures)")
    ap.add_argument("--profile-decode", type=int, default=0, metavar="M",
                    help="only decode steps of the gate/up shape at this M (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep()
    if args.profile_decode:
        return run_profile_decode(args)
    if args.profile_layer:
        return run_profile_layer(args)
    if args.gac_sweep:
        return run_gac_sweep(args)
    return run_ours(args)


def run_profile_decode(args):
    """Decode steps of the gate/up shape (K 4096, r 2867, N 14336) at M =
    args.profile_decode, for ncu captures of this command: warmup + steps
    calls on one set of inputs, no timing line."""
    import torch
    import rank_linear_layers_b200 as lr
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    _, dk, dr, dn = DECODE_SHAPES[0]
    dm = args.profile_decode
    q = lrgen.lowrank_problem(dm, dk, dr, dn, seed=0)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    Xd, Ad, Bd = to_dev(q["X"]), to_dev(q["A"]), to_dev(q["B"])
    Yd = torch.empty((dm, dn), dtype=torch.bfloat16, device=dev)
    launches0 = lr.kernel_launch_count()
    for _ in range(args.warmup + args.steps):
        lr.lr_linear(Xd, Ad, Bd, None, Y=Yd)
    torch.cuda.synchronize()
    status = lr.last_device_status()
    print(json.dumps({"profile_run": "decode", "M": dm, "K": dk, "r": dr, "N": dn,
                      "gpu_launches": int(lr.kernel_launch_count() - launches0),
                      "status": int(status)}))
    return 0 if status == lr.LR_OK else 1


def run_profile_layer(args):
    """The Llama-3-8B decoder layer at M = 1 through lr_linear_group (one
    streamed launch per call; seed 7, N_int 14336), warmup + steps calls,
    for ncu captures of this command; no timing line."""
    import torch
    import rank_linear_layers_b200 as lr
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    n_int = 14336
    layer = lrgen.decoder_layer(1, seed=7, n_int=n_int)
    xs = {k: _dev_bits(v, dev) for k, v in layer["inputs"].items()}
    packed = torch.empty((1, 2 * n_int), dtype=torch.bfloat16, device=dev)
    entries = []
    for name, p in layer["projs"].items():
        e = dict(X=xs[p["x"]], A=_dev_bits(p["A"], dev), B=_dev_bits(p["B"], dev), K=p["K"],
                 r=p["r"], N=p["N"])
        if name in ("gate", "up"):
            e["Y_ptr"] = packed.data_ptr() + (0 if name == "gate" else 2 * n_int)
            e["ld_y"] = 2 * n_int
        else:
            e["Y"] = torch.empty((1, p["N"]), dtype=torch.bfloat16, device=dev)
        entries.append(e)
    launches0 = lr.kernel_launch_count()
    for _ in range(args.warmup + args.steps):
        lr.lr_linear_group(entries, 1)
    torch.cuda.synchronize()
    status = lr.last_device_status()
    print(json.dumps({"profile_run": "layer", "M": 1, "ranks": layer["ranks"],
                      "gpu_launches": int(lr.kernel_launch_count() - launches0),
                      "status": int(status)}))
    return 0 if status == lr.LR_OK else 1


def run_gac_sweep(args):
    """The GAC planner's dimension sweep (§4.2 of the GAC paper) on this GPU:
    for each weight shape of the 32-layer Llama-3-8B-shaped model, the time
    per lr_linear call at every rank the planner may choose, M = args.gac_m
    tokens.  One JSON line: {"times_us": {"KxN": {rank: us}}}, the input of
    ``python -m rank_linear_layers_b200.gac --times``.  X rotates over copies
    larger than twice L2; A and B of a rank are the leading columns / rows of
    one seeded draw."""
    import torch
    import rank_linear_layers_b200 as lr
    from rank_linear_layers_b200 import gac
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    ws = [gac.Weight(**d) for d in lrgen.gac_model(32, seed=11)]
    Mw = args.gac_m
    out = {}
    for (Kw, Nw), ranks in sorted(gac.sweep_plan(ws).items()):
        rmax = max(ranks)
        X0 = _dev_bits(lrgen.normal_bf16(0, 1, (Mw, Kw)), dev)
        Xs = [X0] + [X0.clone() for _ in range(max(1, math.ceil(2 * l2 / (X0.numel() * 2))))]
        Af = _dev_bits(lrgen.normal_bf16(0, 2, (Kw, rmax), 1.0 / math.sqrt(Kw)), dev)
        Bf = _dev_bits(lrgen.normal_bf16(0, 3, (rmax, Nw), 1.0 / math.sqrt(rmax)), dev)
        Y = torch.empty((Mw, Nw), dtype=torch.bfloat16, device=dev)
        t = {}
        for r in ranks:
            A = Af[:, :r].contiguous()
            B = Bf[:r].contiguous()

            def st(i, A=A, B=B):
                lr.lr_linear(Xs[i % len(Xs)], A, B, None, Y=Y)
            t[r] = round(time_steps(st, 20, 3) / 20 * 1e6, 3)
        out[f"{Kw}x{Nw}"] = t
        del Xs, Af, Bf, Y
    status = lr.last_device_status()
    print(json.dumps({"gac_sweep": True, "M": Mw, "times_us": out, "status": int(status)}))
    return 0 if status == lr.LR_OK else 1


def run_sweep():
    """The full misalignment sweep (M = K = N = 4096), one JSON line."""
    import torch
    import rank_linear_layers_b200 as lr
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    ranks = list(range(1000, 1101)) + [64, 128, 512, 2048]
    t = sweep_times(lr, dev, l2, ranks)
    peaks = load_peaks()
    rows = {}
    worst = 0.0
    for r in range(1000, 1101):
        if r % 8 == 0:
            continue
        lo, hi = r - r % 8, r - r % 8 + 8
        near = [n for n in ([lo] if r % 8 < 4 else ([hi] if r % 8 > 4 else [lo, hi])) if n in t]
        d = max(t[r]["ps_per_flop"] / t[n]["ps_per_flop"] - 1.0 for n in near)
        rows[r] = round(d * 100, 2)
        worst = max(worst, d)
    roof = {}
    for r in ranks:
        rf = acc.roofline(acc.flops(4096, 4096, r, 4096), acc.algorithmic_bytes(4096, 4096, r, 4096),
                          peaks["bf16_tflops"], peaks["hbm_gbs"])
        roof[r] = round(rf.t_roof_s / (t[r]["us"] * 1e-6), 3)
    print(json.dumps({"sweep": "M=K=N=4096", "us": {r: round(v["us"], 2) for r, v in t.items()},
                      "frac_roofline": roof, "pct_slower_than_nearest_aligned_per_flop": rows,
                      "worst_pct": round(worst * 100, 2), "target_pct": 5.0}))
    return 0


if __name__ == "__main__":
    sys.exit(main())

"""The C-ABI library loads and exports every declared symbol (no GPU needed),
and argument errors come back before any CUDA call."""
import ctypes
import os
import re

import pytest

import rank_linear_layers_b200 as lr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(lr_[a-z_0-9]+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def L():
    from rank_linear_layers_b200 import build
    if build.needs_build():
        build.build()
    return lr.lib()


def test_exports_every_declared_symbol(L):
    declared = _declared()
    assert declared, "no declarations found"
    for name in declared:
        assert hasattr(L, name), f"missing export {name}"
    assert declared == set(lr.EXPORTS)


def test_status_strings(L):
    assert lr.status_string(lr.LR_OK) == "LR_OK"
    assert lr.status_string(lr.LR_ERR_TIMEOUT) == "LR_ERR_TIMEOUT"
    assert lr.status_string(99) == "LR_ERR_UNKNOWN"


def test_invalid_arguments_rejected_before_cuda(L):
    p = ctypes.c_void_p(0x1000)
    # Negative sizes.
    assert L.lr_linear(p, p, p, None, p, -1, 4, 4, 4, None) == lr.LR_ERR_INVALID_ARG
    assert L.lr_linear(p, p, p, None, p, 4, 4, -3, 4, None) == lr.LR_ERR_INVALID_ARG
    # Null inputs with a nonempty problem.
    assert L.lr_linear(None, p, p, None, p, 4, 4, 4, 4, None) == lr.LR_ERR_INVALID_ARG
    assert L.lr_linear(p, p, p, None, None, 4, 4, 4, 4, None) == lr.LR_ERR_INVALID_ARG
    # Odd (not 2-byte aligned) pointer.
    assert L.lr_linear(ctypes.c_void_p(0x1001), p, ctypes.c_void_p(0x9000), None,
                       ctypes.c_void_p(0x20000), 4, 4, 4, 4, None) == lr.LR_ERR_INVALID_ARG
    # Y overlapping X.
    assert L.lr_linear(ctypes.c_void_p(0x1000), ctypes.c_void_p(0x8000), ctypes.c_void_p(0x9000),
                       None, ctypes.c_void_p(0x1004), 4, 4, 4, 4, None) == lr.LR_ERR_INVALID_ARG
    # Sizes past int32 are unsupported.
    assert L.lr_linear(p, p, p, None, p, 1 << 31, 4, 4, 4, None) == lr.LR_ERR_UNSUPPORTED
    # Empty problems are a no-op that needs no device.
    assert L.lr_linear(None, None, None, None, None, 0, 4, 4, 4, None) == lr.LR_OK
    assert L.lr_linear(None, None, None, None, None, 4, 4, 4, 0, None) == lr.LR_OK
    # Group: bad count, and two projections writing the same elements.
    assert L.lr_linear_group(None, -1, 4, None) == lr.LR_ERR_INVALID_ARG
    arr = (lr.LrProj * 2)()
    for i in range(2):
        arr[i] = lr.LrProj(0x100000, 8, 0x200000, 0x300000, None, 0x400000, 16, 4, 16)
    assert L.lr_linear_group(arr, 2, 4, None) == lr.LR_ERR_INVALID_ARG


def test_packed_halves_are_accepted_by_validation(L):
    # gate and up write the two halves of one [M, 2N] buffer: disjoint, valid.
    # Validation passes; without a device the call then fails on CUDA, not on
    # the arguments.
    arr = (lr.LrProj * 2)()
    N = 12203
    arr[0] = lr.LrProj(0x100000, 8, 0x200000, 0x300000, None, 0x4000000, 2 * N, 4, N)
    arr[1] = lr.LrProj(0x100000, 8, 0x210000, 0x310000, None, 0x4000000 + 2 * N, 2 * N, 4, N)
    assert L.lr_linear_group(arr, 2, 3, None) != lr.LR_ERR_INVALID_ARG
    # Shift the second half left by one element: now they share a column.
    arr[1] = lr.LrProj(0x100000, 8, 0x210000, 0x310000, None, 0x4000000 + 2 * N - 2, 2 * N, 4, N)
    assert L.lr_linear_group(arr, 2, 3, None) == lr.LR_ERR_INVALID_ARG


def test_silu_gate_validation(L):
    """A gate must be another projection of the group, with the same N and
    no gate of its own; checked before anything reaches the device."""
    def group(gates, ns=(16, 16, 16)):
        arr = (lr.LrProj * len(ns))()
        for i, (n, g) in enumerate(zip(ns, gates)):
            arr[i] = lr.LrProj(0x100000, 8, 0x200000 + i * 0x10000, 0x300000 + i * 0x10000, None,
                               0x4000000 + i * 0x100000, n, 4, n, 0, g)
        return L.lr_linear_group(arr, len(ns), 3, None)
    for bad in [(0, 4, 0),      # gate index past the group
                (0, 2, 0),      # its own gate
                (2, 1, 0),      # the gate has a gate
                (0, -1, 0)]:    # negative
        assert group(bad) == lr.LR_ERR_INVALID_ARG, bad
    assert group((0, 1, 0), ns=(16, 24, 16)) == lr.LR_ERR_INVALID_ARG  # N differs
    # A valid group gets past validation (then needs a device).
    assert group((0, 1, 0)) != lr.LR_ERR_INVALID_ARG


def test_controls(L):
    assert L.lr_set_path(7) == lr.LR_ERR_INVALID_ARG
    assert L.lr_set_path(0) == lr.LR_OK
    assert L.lr_set_wait_limit_ns(-1) == lr.LR_ERR_INVALID_ARG
    assert L.lr_set_wait_limit_ns(0) == lr.LR_OK
    assert L.lr_kernel_launch_count() >= 0
    # Tile width: 0 (automatic) or a multiple of 32 up to 256.
    for bad in (-32, 16, 48, 257, 288):
        assert L.lr_set_tile_n(bad) == lr.LR_ERR_INVALID_ARG
    for ok in (32, 96, 256, 0):
        assert L.lr_set_tile_n(ok) == lr.LR_OK
    for bad in (-1, 2, 3):
        assert L.lr_set_split_k(bad) == lr.LR_ERR_INVALID_ARG
    assert L.lr_set_split_k(0) == lr.LR_OK and L.lr_set_split_k(1) == lr.LR_OK
    for bad in (-1, 3):
        assert L.lr_set_t_precision(bad) == lr.LR_ERR_INVALID_ARG
    for ok in (1, 2, 0):
        assert L.lr_set_t_precision(ok) == lr.LR_OK
    for bad in (-1, 2):
        assert L.lr_set_early_copy(bad) == lr.LR_ERR_INVALID_ARG
    assert L.lr_set_early_copy(0) == lr.LR_OK and L.lr_set_early_copy(1) == lr.LR_OK
    assert L.lr_set_withhold_first_stage(2) == lr.LR_ERR_INVALID_ARG
    assert L.lr_set_withhold_first_stage(0) == lr.LR_OK


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError):
        lr.lib(str(tmp_path / "missing.so"))


def test_header_is_plain_c_and_links(L, tmp_path):
    """include/lr_linear.h compiles as C99 (-pedantic) and a C program links
    against the library and calls it (the host-only planner entry point, so
    no GPU is needed)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(
        '#include "lr_linear.h"\n'
        "int main(void) {\n"
        "  int n_cand[2] = {2, 1}; int64_t cost[3] = {8, 16, 24};\n"
        "  double score[2] = {1.0, 1.0}; int64_t base[2] = {8, 24};\n"
        "  int choice[2] = {-1, -1}; double obj = 0.0; lr_proj p = {0}; (void)p;\n"
        "  if (lr_gac_select(2, n_cand, cost, score, base, 40, 8, choice, &obj) != LR_OK) return 2;\n"
        "  return (choice[0] == 1 && choice[1] == 0 && obj == 8.0) ? 0 : 3;\n"
        "}\n")
    libdir = os.path.join(ROOT, "rank_linear_layers_b200")
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-L", libdir, "-llrlinear",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    assert subprocess.run([str(exe)]).returncode == 0


def test_lr_proj_layout_matches_the_binding(tmp_path):
    """The binding's ctypes lr_proj has the C struct's size and field offsets
    (a mismatch would pass the wrong silu_gate or y_f32 silently)."""
    import ctypes
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    fields = [name for name, _ in lr.LrProj._fields_]
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stddef.h>\n#include <stdio.h>\n#include "lr_linear.h"\n'
        "int main(void) {\n"
        '  printf("%zu", sizeof(lr_proj));\n'
        + "".join(f'  printf(" %zu", offsetof(lr_proj, {f}));\n' for f in fields)
        + '  printf("\\n");\n  return 0;\n}\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    want = [ctypes.sizeof(lr.LrProj)] + [getattr(lr.LrProj, f).offset for f in fields]
    assert got == want


def test_prepare_factor_layout():
    """prepare_factor: the same values, rows at the library's factor pitch
    (columns rounded up to 64), unit column stride (host code and the
    library's pitch rule; no GPU)."""
    import torch
    for rows, cols in [(5, 107), (3, 64), (2, 1), (4, 1741)]:
        W = torch.randn(rows, cols).bfloat16()
        V = lr.prepare_factor(W)
        assert tuple(V.shape) == (rows, cols) and V.stride(1) == 1
        assert V.stride(0) == lr.factor_pitch(cols) == -(-cols // 64) * 64
        assert torch.equal(V, W)

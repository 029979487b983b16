"""The streamed decode kernel's work split, checked on the host (no GPU):
block widths (multiples of 8, at most 248, the fewest blocks), every row of
every column block of every projection taken by exactly one CTA, phase-0
pieces listed before phase-1 pieces, a CTA's share within two rows of an
even split, and the one-block form (stream_piece) equal to the list form
(stream_segments).  The shared header functions are compiled with nvcc
into a host program (tests/stream_plan_check.cu)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_stream_work_split(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    exe = tmp_path / "stream_plan_check"
    subprocess.run([nvcc, "-std=c++17", "-O2", "--expt-relaxed-constexpr",
                    "-I", os.path.join(ROOT, "rank_linear_layers_b200", "csrc"),
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "stream_plan_check.cu"), "-o", str(exe)],
                   check=True, capture_output=True, timeout=600)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip().endswith("OK")

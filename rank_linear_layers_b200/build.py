"""Build liblrlinear.so (the CUDA library behind include/lr_linear.h) in-tree.

    python -m rank_linear_layers_b200.build

nvcc compiles every .cu under csrc/ for sm_100a only (B200); the CUDA runtime
is linked statically, so the library needs no libcudart at run time and
loads on a machine without a GPU (its entry points then fail with an error
code instead of computing).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "liblrlinear.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3", "--expt-relaxed-constexpr",
         "-cudart", "static"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def needs_build(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps += glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(out: str = LIB, verbose: bool = False, extra=()) -> str:
    """Compile csrc/*.cu into one shared library (about a minute)."""
    cmd = [nvcc(), *ARCH, *FLAGS, "-shared", "-I", INCLUDE, *extra, *sources(), "-o", out + ".tmp"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    build(verbose=True, extra=sys.argv[1:])
    print(LIB)

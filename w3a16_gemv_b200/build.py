"""Build libw3a16.so in-tree with nvcc for sm_100a (B200).

``python -m w3a16_gemv_b200.build`` or ``build()`` from Python.  The library is
one translation unit (``csrc/api.cu`` includes the kernels) linked against the
static CUDA runtime, so it does not depend on torch's copy of libcudart.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libw3a16.so")
HEADER = os.path.join(ROOT, "include", "w3a16.h")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared", "--expt-relaxed-constexpr"]


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh"))) + [HEADER]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libw3a16.so")


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, out: str | None = None, defines=()) -> str:
    """Compile the library if it is missing or older than its sources; return its path.

    `out` and `defines` (e.g. ``["W3_DECODE_DEPTH=3"]``) build a variant elsewhere,
    for tuning sweeps; the default build uses the constants in the sources."""
    target = out or LIB
    if not force and out is None and up_to_date():
        return LIB
    tmp = target + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH_FLAGS, *NVCC_FLAGS, *[f"-D{d}" for d in defines], "-o", tmp,
           os.path.join(CSRC, "api.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))

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


def up_to_date(path: str = LIB) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, out: str | None = None, defines=()) -> str:
    """Compile the library if it is missing or older than its sources; return its path.

    `out` and `defines` build a variant of the library elsewhere: the failure-detection
    test builds one with ``W3_TEST_HOOKS`` (a test-only kernel that makes a bounded wait run
    out) and a short ``W3_WAIT_LIMIT_CYCLES``.  The product build has neither."""
    target = out or LIB
    if not force and up_to_date(target):
        return target
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

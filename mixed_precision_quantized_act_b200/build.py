"""Builds the in-tree CUDA library ``libmixllm_b200.so`` for sm_100a with nvcc.

The library is one translation unit (``csrc/mixllm.cu``) that exports the C ABI
of ``include/mixllm.h``; the CUDA runtime is linked statically and the driver's
tensor-map encoder is looked up at run time, so loading the library needs no
GPU.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmixllm_b200.so")
# The checked build: every tensor- and shared-memory access of the GEMM
# kernels range-checked first (MIXLLM_CHECKED=1); for tests, not for speed.
LIB_CHECKED = os.path.join(HERE, "libmixllm_b200_checked.so")
MAIN = os.path.join(HERE, "csrc", "mixllm.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
]


def _sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*"))) + [os.path.join(ROOT, "include", "mixllm.h")]


def needs_build(checked: bool = False) -> bool:
    lib = LIB_CHECKED if checked else LIB
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    if not force and not needs_build(checked):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *(["-DMIXLLM_CHECKED=1"] if checked else []),
           *(["-Xptxas", "-v"] if verbose else []), "-o", tmp, MAIN]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, checked="--checked" in sys.argv))

"""Build libzero.so (the CUDA library) in-tree for sm_100a.

Usage: python zero_sharded_optimizer_03_b200/build.py  (nvcc cross-compiles; no GPU needed).
Run it as a script (or load it by path): importing it through the package would first load
the library it is meant to (re)build.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
SO = os.path.join(HERE, "libzero.so")
SOURCES = ["zero_abi.cu", "zero_accounting.cpp", "zero_host_adam.cpp"]
DEPS = SOURCES + ["zero_kernels.cuh", "zero_tma.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-fmad=false",                      # every fp32/fp64 operation rounds on its own
    "-Xcompiler", "-fPIC,-ffp-contract=off,-fno-math-errno",
    "-Xptxas", "-v",
    "-shared",
]


def nvcc() -> str:
    return os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")


def stale() -> bool:
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    deps = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(INCLUDE, "zero.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return SO
    tmp = SO + ".tmp.%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, *[os.path.join(CSRC, s) for s in SOURCES],
           "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libzero.so")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    build(force=True, verbose=True)
    print(SO)

"""Build libsvdq.so in-tree for sm_100a (nvcc + the host C++ compiler).

    python -m w4a4_rank_corrected_b200.build [--verbose]

The library is plain C ABI (include/svdq.h): device code is compiled for
sm_100a only, the CUDA runtime is linked statically, and the driver entry
point used for TMA descriptors is looked up at run time, so the library
loads on a machine without a GPU driver (its GPU calls then report
SVDQ_ERR_UNSUPPORTED_ARCH).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libsvdq.so")
SOURCES = [os.path.join(HERE, "csrc", "svdq_api.cu"), os.path.join(HERE, "csrc", "pack.cpp")]
DEPS = SOURCES + [os.path.join(HERE, "csrc", f) for f in
                  ("ptx.cuh", "quantize_act.cuh", "quantize_act64.cuh", "w4a4_gemm.cuh",
                   "gelu.cuh", "row_scales.cuh", "awq_gemv.cuh")] + \
       [os.path.join(ROOT, "include", "svdq.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(verbose_ptxas: bool = False):
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
           "-std=c++17", "--shared", "-cudart", "static",
           "-Xcompiler", "-fPIC,-fopenmp,-ffp-contract=off,-mavx2",
           "-I", os.path.join(ROOT, "include")]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", LIB] + SOURCES + ["-lgomp"]
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = command(verbose_ptxas=verbose)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed building libsvdq.so")
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)

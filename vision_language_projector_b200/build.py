"""Build ``libvlproj.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: ``python vision_language_projector_b200/build.py [--force] [--verbose]`` (run it
as a script: importing the package would load the library being built).
The library links the CUDA runtime statically and reaches the driver's
tensor-map encoder through the runtime's entry-point query, so it needs no
link-time libcuda and loads on machines without a GPU.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libvlproj.so")
SOURCES = [os.path.join(CSRC, f) for f in ("vlproj.cu", "vlproj_backward.cu", "vlproj_host.cu", "vlproj_noalloc.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("ptx.cuh", "gemm_sm100.cuh", "kernels_aux.cuh", "kernels_bwd.cuh", "host.cuh", "gelu_poly.cuh")] + [
    os.path.join(ROOT, "include", "vlproj.h")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB, verbose: bool = False) -> list:
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "--expt-relaxed-constexpr", "-shared", "-Xcompiler", "-fPIC,-O2", "-I", os.path.join(ROOT, "include"),
           "-o", out] + SOURCES
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, verbose: bool = False) -> str:
    stale = not os.path.exists(LIB) or any(os.path.getmtime(d) > os.path.getmtime(LIB) for d in DEPS)
    if force or stale:
        tmp = LIB + ".tmp"
        subprocess.check_call(command(tmp, verbose))
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)

"""Builds libfa_b200.so in-tree with nvcc for sm_100a.

Usage: python exact_io_aware_90_b200/build.py [--verbose-ptxas]   (by path: importing the package would load the
existing library first)
The library lands next to this file; the Python binding loads it from there.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB_NAME = "libfa_b200.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
SOURCES = ["libfa_b200.cu"]
DEPS = ["fa_api.cu", "fa_fwd.cu", "fa_bwd.cu", "fa_decode.cu", "fa_merge.cu", "fa_noalloc.cu"]
HEADERS = ["fa_internal.h", "sm100.cuh", os.path.join("..", "..", "include", "fa.h")]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put the CUDA toolkit on PATH")


def needs_rebuild() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    deps = [os.path.join(CSRC, f) for f in SOURCES + DEPS + HEADERS] + [__file__]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(verbose_ptxas: bool = False, force: bool = False) -> str:
    if not force and not needs_rebuild():
        return LIB_PATH
    cmd = [
        nvcc_path(),
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared",
        "--expt-relaxed-constexpr",
        "-I", os.path.join(ROOT, "include"),
        "-o", LIB_PATH + ".tmp",
    ] + [os.path.join(CSRC, f) for f in SOURCES]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building " + LIB_NAME)
    if verbose_ptxas:
        sys.stderr.write(res.stderr)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(verbose_ptxas="--verbose-ptxas" in sys.argv, force=True))

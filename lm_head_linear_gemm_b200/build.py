"""Build the in-tree C-ABI library ``libflce.so`` for sm_100a with nvcc.

    python -m lm_head_linear_gemm_b200.build [--verbose-ptxas]
    FLCE_BUILD_DEFINES="-DFLCE_DW_GROUPS=2" python -m lm_head_linear_gemm_b200.build --force

The library is written next to this file so that it travels with the source tree;
nothing is installed into site-packages.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB_PATH = os.path.join(HERE, "libflce.so")
SOURCES = [os.path.join(CSRC, "flce_api.cu")]
HEADERS = [os.path.join(CSRC, f) for f in ("sm100.cuh", "gemm.cuh", "rowwise.cuh")] + [
    os.path.join(ROOT, "include", "flce.h")]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA 12.9 toolkit is required to build libflce.so")


def nvcc_flags(verbose_ptxas: bool = False) -> list[str]:
    flags = [
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared",
        "--expt-relaxed-constexpr",
        "-I", os.path.join(ROOT, "include"),
    ]
    if verbose_ptxas:
        flags += ["-Xptxas", "-v"]
    # build-time tuning constants of flce_api.cu (e.g. "-DFLCE_DW_GROUPS=2"), for measurements
    flags += os.environ.get("FLCE_BUILD_DEFINES", "").split()
    return flags


def is_stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS)


def build(force: bool = False, verbose_ptxas: bool = False, quiet: bool = False) -> str:
    if not force and not is_stale():
        return LIB_PATH
    tmp = LIB_PATH + ".tmp"
    cmd = [nvcc_path()] + nvcc_flags(verbose_ptxas) + ["-o", tmp] + SOURCES
    if not quiet:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose_ptxas or (res.stderr.strip() and not quiet):
        print(res.stderr, file=sys.stderr)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))

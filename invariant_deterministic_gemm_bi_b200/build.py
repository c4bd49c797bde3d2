"""Build libbigemm.so in-tree with nvcc for sm_100a.

Usage: ``python -m invariant_deterministic_gemm_bi_b200.build [--verbose]``.

The numerics-relevant flags are fixed here: no fast-math, no flush-to-zero, IEEE division and
square root, and no automatic FMA contraction (the kernels spell out every fused multiply-add
they want).  No environment variable changes them.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
REPO = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
SOURCES = [os.path.join(CSRC, "bi_gemm.cu"), os.path.join(CSRC, "bi_moe.cu"),
           os.path.join(CSRC, "bi_attention.cu"), os.path.join(CSRC, "bi_quantize.cu")]
HEADERS = [os.path.join(CSRC, "bi_kernels.cuh"), os.path.join(CSRC, "bi_kernels_pair.cuh"),
           os.path.join(CSRC, "ptx_sm100.cuh"), os.path.join(REPO, "include", "bi_gemm.h"),
           os.path.join(REPO, "include", "bi_moe.h"), os.path.join(REPO, "include", "bi_attention.h"),
           os.path.join(REPO, "include", "bi_quantize.h")]
LIB = os.path.join(PKG, "libbigemm.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=false",
    "-cudart", "static",
]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [nvcc_path(), *NVCC_FLAGS, "-I", os.path.join(REPO, "include")]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    tmp = LIB + ".tmp"
    cmd += SOURCES + ["-o", tmp]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        sys.stderr.write(proc.stdout + proc.stderr)
        raise RuntimeError("nvcc failed building libbigemm.so")
    if verbose:
        sys.stderr.write(proc.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))

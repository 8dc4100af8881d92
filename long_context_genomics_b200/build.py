"""Build libag.so (the CUDA kernels and the C ABI) in-tree for sm_100a.

    python long_context_genomics_b200/build.py [--verbose] [--ptxas-v]

The library links the CUDA runtime statically and reaches the driver's
tensor-map encoder through cudaGetDriverEntryPoint, so it needs no CUDA
driver library at link time and cross-compiles on a machine without a GPU.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libag.so")
SOURCES = ["ag_api.cu", "attn_fwd_sm100.cu", "attn_noalloc.cu", "attn_bwd.cu",
           "attn_bwd_sm100.cu", "pair_bias_project.cu"]
HEADERS = ["sm100.cuh", "ag_internal.h", "attn_bwd_phases.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _inputs():
    return ([os.path.join(CSRC, s) for s in SOURCES + HEADERS]
            + [os.path.join(ROOT, "include", "ag.h")])


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(verbose: bool = False, ptxas_v: bool = False) -> str:
    cmd = [
        NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
        "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
        "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"),
        "-o", LIB,
    ] + [os.path.join(CSRC, s) for s in SOURCES]
    if ptxas_v:
        cmd[1:1] = ["-Xptxas", "-v"]
    if verbose:
        print(" ".join(cmd))
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("libag build failed:\n" + res.stdout + res.stderr)
    if verbose or ptxas_v:
        sys.stdout.write(res.stdout + res.stderr)
    return LIB


def ensure_built() -> str:
    if needs_build():
        build()
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true")
    a = ap.parse_args()
    print(build(verbose=a.verbose, ptxas_v=a.ptxas_v))

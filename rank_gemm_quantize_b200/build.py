"""Builds libsvdq.so in-tree with nvcc for sm_100a.

    python -m rank_gemm_quantize_b200.build [--verbose]

The library is the whole product: the CUDA kernels and the C ABI of
include/svdq.h. It links the CUDA runtime and cuSOLVER (float64 SVD in the
offline prepare step) and resolves the tensor-map encoder through the runtime's
driver entry point, so it needs no libcuda at link time.
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
INCLUDE = os.path.join(ROOT, "include")
OUT = os.path.join(HERE, "libsvdq.so")
SOURCES = ["svdq_api.cu", "act_quant.cu", "gemm_nvfp4.cu", "gemm_int4.cu", "prepare_kernels.cu", "noalloc.cu",
           "w4a16.cu"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
         "-Xcompiler", "-fvisibility=hidden", "-DSVDQ_BUILD"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = OUT, extra=()) -> list[str]:
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    return [nvcc(), *ARCH, *FLAGS, "-I", INCLUDE, "-I", CSRC, *extra, "-o", out, *srcs, "-lcusolver", "-lcudart"]


def build(verbose: bool = False, force: bool = False) -> str:
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "svdq.h")]
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= max(os.path.getmtime(d) for d in deps):
        return OUT
    cmd = command()
    if verbose:
        print(" ".join(cmd), flush=True)
    tmp = OUT + ".tmp"
    cmd[cmd.index("-o") + 1] = tmp
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libsvdq.so")
    if verbose and (res.stdout or res.stderr):
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(verbose=a.verbose, force=a.force))

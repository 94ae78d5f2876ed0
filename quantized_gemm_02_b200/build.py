"""Builds libhq.so (sm_100a) in-tree with nvcc.

    python -m quantized_gemm_02_b200.build [--verbose]

The library is one translation unit (csrc/libhq.cu) compiled for
``arch=compute_100a,code=sm_100a`` with line info, linked against the CUDA
runtime.  The output lands next to this file so that it travels with the
source tree.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libhq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = sources() + [os.path.join(HERE, "..", "include", "hq.h")]
    return all(os.path.getmtime(s) <= t for s in deps)


def build(verbose: bool = False, force: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [
        NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
        "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
        "-I", os.path.join(HERE, "..", "include"),
        "-cudart", "static", "-o", LIB + ".tmp", os.path.join(CSRC, "libhq.cu"),
    ]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=not verbose, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + (r.stdout or "") + (r.stderr or ""))
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
    print(LIB)

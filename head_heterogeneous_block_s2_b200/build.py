"""Build libs2attn.so in-tree with nvcc for sm_100a.

    python -m head_heterogeneous_block_s2_b200.build [--verbose]

The CUDA runtime is linked statically and the driver is reached through
cudaGetDriverEntryPoint, so the library loads (and its symbols can be listed)
on a machine without a GPU.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libs2attn.so")

SOURCES = [os.path.join(CSRC, "s2attn.cu"), os.path.join(CSRC, "layout.cpp")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("ptx.cuh", "store.cuh", "umma.cuh", "lists.cuh", "prefill_pair_sm100.cuh", "backward_sm100.cuh", "chunk_sm100.cuh", "decode.cuh")] + [
    os.path.join(INCLUDE, "s2attn.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]


def nvcc() -> str:
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cand = os.path.join(cuda, "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", tmp, *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)

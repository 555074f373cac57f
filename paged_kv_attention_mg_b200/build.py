"""Builds libmg.so (the CUDA library behind include/mg.h) in-tree for sm_100a.

    python -m paged_kv_attention_mg_b200.build [--force]

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically and reaches the driver API only through cudaGetDriverEntryPoint,
so it needs no libcuda at link time.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libmg.so")
MAIN = os.path.join(CSRC, "mg.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def _sources():
    out = [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    out += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh"))]
    return out


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build_library(force: bool = False, verbose: bool = False, output: str = LIBRARY,
                  extra_flags=()) -> str:
    if not force and os.path.exists(output):
        newest = max(os.path.getmtime(s) for s in _sources())
        if os.path.getmtime(output) >= newest:
            return output
    tmp = output + ".tmp%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, *extra_flags, "-I" + INCLUDE, "-o", tmp, MAIN]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, output)
    return output


if __name__ == "__main__":
    build_library(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIBRARY)

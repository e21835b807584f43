"""Build libexternd.so in-tree for B200 (sm_100a) with nvcc.

Usage: python -m ternary_rank_weight_b200.build
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCES = [os.path.join(HERE, "csrc", name) for name in ("externd.cu", "externd_nt1024.cu", "infer.cu")]
DEPS = SOURCES + [os.path.join(HERE, "csrc", name) for name in ("externd_kernels.cuh", "als_cluster.cuh", "block_als.cuh")] \
    + [os.path.join(ROOT, "include", "externd.h")]
OUT = os.path.join(HERE, "libexternd.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    # the block ALS (§2.4) hands its plain fp64 GEMMs and Cholesky solves to the vendor libraries
    "-lcublas", "-lcusolver", "-Xlinker", "-rpath=/usr/local/cuda/lib64",
]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return OUT
    tmp = OUT + ".tmp"
    cmd = [nvcc_path(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), *SOURCES, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))

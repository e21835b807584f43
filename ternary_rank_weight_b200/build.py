"""Build libexternd.so in-tree for B200 (sm_100a) with nvcc.

Usage: python -m ternary_rank_weight_b200.build
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
# externd_nt256.cu and externd_nt1024.cu compile the ALS machinery of externd.cu at other block sizes
SOURCES = [os.path.join(HERE, "csrc", name) for name in ("externd.cu", "externd_nt256.cu", "externd_nt1024.cu", "infer.cu")]
DEPS = SOURCES + [os.path.join(HERE, "csrc", name) for name in ("externd_kernels.cuh", "als_cluster.cuh", "block_als.cuh")] \
    + [os.path.join(ROOT, "include", "externd.h")]
OUT = os.path.join(HERE, "libexternd.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = [*ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC"]
LINK_FLAGS = [
    *ARCH_FLAGS, "-shared",
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
    """Compile every source to an object (in parallel: one nvcc per source), then link."""
    if not force and not needs_build():
        return OUT
    tmp = OUT + ".tmp"
    with tempfile.TemporaryDirectory(prefix="externd_build_") as objdir:
        objs, procs = [], []
        for src in SOURCES:
            obj = os.path.join(objdir, os.path.basename(src) + ".o")
            cmd = [nvcc_path(), *COMPILE_FLAGS, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd), flush=True)
            objs.append(obj)
            procs.append((cmd, subprocess.Popen(cmd)))
        failed = [cmd for cmd, p in procs if p.wait() != 0]
        if failed:
            raise subprocess.CalledProcessError(1, failed[0])
        subprocess.run([nvcc_path(), *LINK_FLAGS, *objs, "-o", tmp], check=True)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))

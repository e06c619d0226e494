"""Build the CUDA library libatomenc.so in-tree (nvcc, sm_100a only).

Run `python -m sparse_windowed_atom_b200.build` or call build(). The library is built
beside this file so that it travels with the source tree.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libatomenc.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    # IEEE float32: no fast-math, subnormals kept (the pages keep subnormal tails)
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=true",
    "-Xcompiler", "-fPIC",
    "-I", os.path.join(ROOT, "include"),
]
OBJ_DIR = os.path.join(HERE, "_build")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        [os.path.join(ROOT, "include", "atomenc.h")]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in deps())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every translation unit of csrc/ (in parallel) and link libatomenc.so."""
    if not force and not stale():
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    srcs = sources()
    objs = [os.path.join(OBJ_DIR, os.path.basename(f)[:-3] + f".{os.getpid()}.o") for f in srcs]
    extra = ["-Xptxas=-v"] if verbose else []
    procs = []
    for src, obj in zip(srcs, objs):
        cmd = [NVCC, *FLAGS, *extra, "-c", "-o", obj, src]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((src, subprocess.Popen(cmd)))
    failed = [src for src, pr in procs if pr.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, f"nvcc ({', '.join(map(os.path.basename, failed))})")
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                           "-Xcompiler", "-fPIC", "-o", tmp, *objs])
    os.replace(tmp, LIB)
    for o in objs:
        os.remove(o)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)

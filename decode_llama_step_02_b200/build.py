"""Builds libl2c.so, the decode-step library, for sm_100a (in-tree)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libl2c.so")
SOURCES = [os.path.join(HERE, "csrc", n) for n in ("l2c.cu", "attention_noalloc.cu")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _inputs():
    return (glob.glob(os.path.join(HERE, "csrc", "*")) + [os.path.join(ROOT, "include", "l2c.h")])


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compiles every source to an object (in parallel), then links the library."""
    if not force and not stale():
        return LIB
    tag = f".tmp{os.getpid()}"
    objs, procs = [], []
    for src in SOURCES:
        obj = os.path.join(HERE, os.path.basename(src) + tag + ".o")
        cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-c", "-o", obj, src]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        objs.append(obj)
        procs.append(subprocess.Popen(cmd))
    try:
        failed = [src for src, p in zip(SOURCES, procs) if p.wait() != 0]
        if failed:
            raise subprocess.CalledProcessError(1, f"nvcc {' '.join(failed)}")
        tmp = LIB + tag
        subprocess.check_call([_nvcc(), *NVCC_FLAGS, "-shared", "-o", tmp, *objs, "-lcudart"])
        os.replace(tmp, LIB)
    finally:
        for o in objs:
            if os.path.exists(o):
                os.remove(o)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])

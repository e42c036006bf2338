"""Builds libcarve.so (the C-ABI library of include/carve.h) in-tree for sm_100a with nvcc.

Each .cu file is compiled to an object in its own process (in parallel), then the objects are
linked into the shared library; an object is rebuilt only when its source, a header or this
file is newer than it."""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libcarve.so")
OBJ = os.path.join(PKG, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2"]


def sources():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cuh"))) + [os.path.join(ROOT, "include", "carve.h"),
                                                                     os.path.abspath(__file__)]


def deps():
    return sources() + headers()


def _obj(src):
    return os.path.join(OBJ, os.path.basename(src)[:-3] + ".o")


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in deps())


def _compile(src, nvcc, force, verbose):
    obj = _obj(src)
    newest = max(os.path.getmtime(p) for p in [src] + headers())
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj
    tmp = obj + f".tmp{os.getpid()}"
    cmd = [nvcc, *FLAGS, *ARCH, "-I", os.path.join(ROOT, "include"), "-c", "-o", tmp, src]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, obj)
    return obj


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    os.makedirs(OBJ, exist_ok=True)
    srcs = sources()
    with ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(lambda s: _compile(s, nvcc, force, verbose), srcs))
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([nvcc, "-shared", *ARCH, "-o", tmp, *objs], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)

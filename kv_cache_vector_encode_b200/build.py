"""Builds libtq.so in-tree (nvcc, sm_100a).

    python -m kv_cache_vector_encode_b200.build        # or build() from Python

Compiles every csrc/*.cu and csrc/*.cpp into one shared library next to this file. The CUDA
runtime is linked statically and the driver API is not linked, so the library loads (and its
host-only entry points work) on a machine without a GPU.
"""
from __future__ import annotations

import concurrent.futures
import glob
import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libtq.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-cudart", "static",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + \
        [os.path.join(INCLUDE, "tq.h")]


def _digest(files):
    h = hashlib.sha256()
    for f in files + _headers() + [__file__]:
        h.update(open(f, "rb").read())
    h.update(" ".join(NVCC_FLAGS).encode())
    return h.hexdigest()


def _compile(src, objdir, force, verbose):
    """Compiles one source unless its object is up to date (same source, headers and flags)."""
    obj = os.path.join(objdir, os.path.basename(src) + ".o")
    stamp = obj + ".sha256"
    dig = _digest([src])
    if not force and os.path.exists(obj) and os.path.exists(stamp) and open(stamp).read() == dig:
        return obj
    cmd = ["nvcc", *NVCC_FLAGS, "-I", INCLUDE, "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    with open(stamp, "w") as f:
        f.write(dig)
    return obj


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libtq.so unless an up-to-date build is present; returns its path. Sources compile in
    parallel, each only when it or a header changed."""
    stamp = LIB + ".sha256"
    dig = _digest(_sources())
    if not force and os.path.exists(LIB) and os.path.exists(stamp) and open(stamp).read() == dig:
        return LIB
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    workers = max(1, min(len(_sources()), os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        objs = list(ex.map(lambda s: _compile(s, objdir, force, verbose), _sources()))
    tmp = LIB + ".tmp"
    cmd = ["nvcc", "-shared", *NVCC_FLAGS, "-o", tmp, *objs]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    with open(stamp, "w") as f:
        f.write(dig)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))

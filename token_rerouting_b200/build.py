"""Build libue.so (the sm_100a CUDA library behind include/ue.h) in place.

    python -m token_rerouting_b200.build [--force] [--verbose]

nvcc cross-compiles for sm_100a without a GPU. The library links the CUDA
runtime statically, so it loads beside any PyTorch build.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libue.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libue")
    return cand


def _compile_one(src, obj, verbose):
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH_FLAGS, "-lineinfo", "-Xcompiler", "-fPIC",
           "-rdc=false", "-I", INCLUDE, "-I", CSRC, "-c", "-o", obj + ".tmp", src]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("libue build failed:\n" + " ".join(cmd) + "\n" + res.stdout +
                           res.stderr)
    if verbose:
        sys.stderr.write(f"== {os.path.basename(src)}\n" + res.stdout + res.stderr)
    os.replace(obj + ".tmp", obj)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every csrc/*.cu for sm_100a (one object per source, in
    parallel, into _build/; a source is recompiled when it or any header is
    newer than its object) and link libue.so."""
    if not force and not verbose and up_to_date():
        return LIB
    from concurrent.futures import ThreadPoolExecutor
    bdir = os.path.join(ROOT, "_build", "libue")
    os.makedirs(bdir, exist_ok=True)
    headers = sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h")))
    newest_header = max((os.path.getmtime(h) for h in headers), default=0.0)
    jobs = []
    objs = []
    for src in sources():
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if (force or verbose or not os.path.exists(obj) or
                os.path.getmtime(obj) < max(os.path.getmtime(src), newest_header)):
            jobs.append((src, obj))
    with ThreadPoolExecutor(max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        list(ex.map(lambda j: _compile_one(j[0], j[1], verbose), jobs))
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH_FLAGS, "-shared", "-o", tmp, *objs]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("libue link failed:\n" + " ".join(cmd) + "\n" + res.stdout +
                           res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)

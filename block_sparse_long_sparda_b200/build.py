"""Build libsparda.so (all CUDA kernels + the C ABI) in-tree for sm_100a.

    python -m block_sparse_long_sparda_b200.build [--force] [--verbose-ptxas]

Each .cu file compiles to its own object (in parallel, under _build/, which
git ignores); an object is rebuilt when its source or any header changed.
The objects are then linked into lib/libsparda.so with the CUDA runtime
linked statically.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
OBJDIR = os.path.join(PKG, "_build")
LIB = os.path.join(LIBDIR, "libsparda.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(CSRC, "*.h"))) + [os.path.join(ROOT, "include", "sparda.h")]


def _obj(src):
    return os.path.join(OBJDIR, os.path.basename(src)[:-3] + ".o")


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(f) > t for f in deps)


def up_to_date() -> bool:
    return not _stale(LIB, sources() + headers())


def _compile(src, verbose_ptxas):
    out = _obj(src)
    tmp = out + ".tmp.%d" % os.getpid()
    cmd = [NVCC, *ARCH, *FLAGS, "-I", os.path.join(ROOT, "include"), "-c", "-o", tmp, src]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, out)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not verbose_ptxas and up_to_date():
        return LIB
    os.makedirs(LIBDIR, exist_ok=True)
    os.makedirs(OBJDIR, exist_ok=True)
    hdrs = headers()
    todo = [s for s in sources()
            if force or verbose_ptxas or _stale(_obj(s), [s] + hdrs)]
    with ThreadPoolExecutor(max_workers=max(1, min(len(todo), os.cpu_count() or 4))) as ex:
        for f in [ex.submit(_compile, s, verbose_ptxas) for s in todo]:
            f.result()
    tmp = LIB + ".tmp.%d" % os.getpid()
    subprocess.check_call([NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp,
                           *[_obj(s) for s in sources()]])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))

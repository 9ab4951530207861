"""Build libdsa.so (all CUDA sources, sm_100a) in-tree with nvcc.

Every source is compiled as a whole program in parallel (objects under `_build/` next to
this file; no relocatable device code, so ptxas applies setmaxnreg register splits), then
one nvcc call links them into the shared library.  The
library links the CUDA runtime statically and reaches the driver API (tensor-map encoding)
through cudaGetDriverEntryPoint, so it loads on a machine without a GPU driver.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libdsa.so")
OBJDIR = os.path.join(HERE, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                 "--expt-relaxed-constexpr"]
LINK_FLAGS = [*ARCH, "-Xcompiler", "-fPIC", "-shared", "-cudart", "static"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(CSRC, "*.h"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]


def _inputs():
    return sources() + _headers()


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _inputs())


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}): {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return r.stderr


def build(verbose: bool = False, extra_flags=None) -> str:
    """Compile every CUDA source into libdsa.so next to this file; returns its path."""
    os.makedirs(OBJDIR, exist_ok=True)
    hdr_time = max(os.path.getmtime(p) for p in _headers())
    jobs = []
    for src in sources():
        obj = os.path.join(OBJDIR, os.path.basename(src)[:-3] + ".o")
        fresh = (not extra_flags and os.path.exists(obj) and
                 os.path.getmtime(obj) > max(os.path.getmtime(src), hdr_time))
        if not fresh:
            jobs.append([nvcc(), *COMPILE_FLAGS, *(extra_flags or []), "-I", INCLUDE, "-c",
                         "-o", obj, src])
    objs = [os.path.join(OBJDIR, os.path.basename(s)[:-3] + ".o") for s in sources()]
    if verbose:
        for j in jobs:
            print(" ".join(j), file=sys.stderr)
    with ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 4))) as ex:
        for err in ex.map(_run, jobs):
            if verbose and err:
                print(err, file=sys.stderr)
    tmp = LIB + ".tmp"
    link = [nvcc(), *LINK_FLAGS, "-o", tmp, *objs]
    if verbose:
        print(" ".join(link), file=sys.stderr)
    _run(link)
    os.replace(tmp, LIB)
    return LIB


def build_if_needed(verbose: bool = False) -> str:
    if is_stale():
        return build(verbose=verbose)
    return LIB


if __name__ == "__main__":
    print(build(verbose=True))

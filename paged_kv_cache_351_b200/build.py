"""Build libpa.so (sm_100a kernels + C ABI + host allocator) in-tree.

    python paged_kv_cache_351_b200/build.py [--force] [--verbose] [--ptxas-info]

(run it by path: it does not import the package, whose import loads the
library it is about to rebuild)

nvcc compiles the single CUDA translation unit for sm_100a only
(``-gencode arch=compute_100a,code=sm_100a``); g++ compiles the host
allocator; nvcc links both with the static CUDA runtime into
``paged_kv_cache_351_b200/libpa.so``, next to this file.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT = os.path.join(HERE, "libpa.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
                     "--expt-relaxed-constexpr", "-I", INCLUDE]
CXX_FLAGS = ["-O2", "-fPIC", "-std=c++17", "-Wall", "-I", INCLUDE]


def _nvcc() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand) and not shutil.which(cand):
        raise RuntimeError("nvcc not found")
    return cand


def _sources():
    srcs = []
    for d in (CSRC, INCLUDE):
        for f in sorted(os.listdir(d)):
            if f.endswith((".cu", ".cuh", ".cpp", ".h")):
                srcs.append(os.path.join(d, f))
    return srcs


def _up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(s) <= t for s in _sources() + [os.path.abspath(__file__)])


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or r.returncode:
        sys.stdout.write(r.stdout)
        sys.stderr.write(r.stderr)
    if r.returncode:
        raise RuntimeError(f"build step failed: {' '.join(cmd[:3])} ...")
    return r


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    """Compile libpa.so if any source is newer; return its path."""
    if not force and not ptxas_info and _up_to_date():
        return OUT
    os.makedirs(BUILD_DIR, exist_ok=True)
    nvcc = _nvcc()
    cu_obj = os.path.join(BUILD_DIR, "pa_api.o")
    cpp_obj = os.path.join(BUILD_DIR, "pa_alloc.o")
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    _run([nvcc, *NVCC_FLAGS, *extra, "-c", os.path.join(CSRC, "pa_api.cu"), "-o", cu_obj], verbose or ptxas_info)
    cxx = os.environ.get("CXX") or "g++"
    _run([cxx, *CXX_FLAGS, "-c", os.path.join(CSRC, "pa_alloc.cpp"), "-o", cpp_obj], verbose)
    tmp = OUT + ".tmp"
    _run([nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, cu_obj, cpp_obj], verbose)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers/spills/smem per kernel")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_info=a.ptxas_info))

"""Build libmsa.so (all CUDA sources, sm_100a) in-tree, next to this file.

    python -m block_sparse_gqa_mean_b200.build [--force] [--verbose] [--debug-bounds]

Objects go to <repo>/_build/; the shared library lands in the package
directory, where the Python binding loads it. nvcc cross-compiles for sm_100a
without a GPU.

--debug-bounds builds the bounds-checked variant instead: the same sources
compiled with -DMSA_DEBUG_BOUNDS (objects in <repo>/_build/debug_bounds/)
into libmsa_debug.so, whose kernels check every index they derive from device
data before the access and report MSA_DEV_BOUNDS instead of faulting. The
binding loads it in place of libmsa.so when MSA_LIBRARY names its path.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmsa.so")
DEBUG_LIB = os.path.join(PKG, "libmsa_debug.so")
DEBUG_BUILD = os.path.join(BUILD, "debug_bounds")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _headers_mtime():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs.append(os.path.join(INCLUDE, "msa.h"))
    return max(os.path.getmtime(h) for h in hs)


def _compile(src, force, verbose, extra, objdir):
    obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
    if (not force and os.path.exists(obj) and
            os.path.getmtime(obj) >= max(os.path.getmtime(src), _headers_mtime())):
        return obj, ""
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return obj, (r.stdout + r.stderr) if verbose else ""


def build(force: bool = False, verbose: bool = False, extra=(), debug_bounds: bool = False) -> str:
    """Compile and link; returns the library path. debug_bounds: the
    bounds-checked variant (libmsa_debug.so)."""
    objdir, lib = (DEBUG_BUILD, DEBUG_LIB) if debug_bounds else (BUILD, LIB)
    extra = list(extra) + (["-DMSA_DEBUG_BOUNDS"] if debug_bounds else [])
    os.makedirs(objdir, exist_ok=True)
    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(lambda s: _compile(s, force, verbose, extra, objdir), srcs))
    objs = [o for o, _ in results]
    for _, log in results:
        if log:
            print(log, file=sys.stderr)
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas resource usage")
    ap.add_argument("--debug-bounds", action="store_true",
                    help="build the bounds-checked libmsa_debug.so instead")
    a = ap.parse_args()
    extra = ["-Xptxas", "-v"] if a.verbose else []
    print(build(force=a.force or a.verbose, verbose=a.verbose, extra=extra,
                debug_bounds=a.debug_bounds))


if __name__ == "__main__":
    main()

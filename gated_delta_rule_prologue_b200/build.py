"""Build ``libkda.so`` in-tree with nvcc for sm_100a.

Usage: ``python gated_delta_rule_prologue_b200/build.py [--debug]`` (run as a script, so
that the package, which loads the library at import, is not imported first).  Every ``csrc/*.cu`` file is compiled to an object under
``_build/`` in parallel and linked into ``gated_delta_rule_prologue_b200/libkda.so``
(CUDA runtime linked statically).  Objects are rebuilt when their source or
any header is newer.
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
BUILD = os.path.join(ROOT, "_build")
BUILD_DEBUG = os.path.join(ROOT, "_build_debug")
LIB = os.path.join(PKG, "libkda.so")
LIB_DEBUG = os.path.join(PKG, "libkda_debug.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


def _stale(obj, src, hdr_mtime):
    if not os.path.exists(obj):
        return True
    m = os.path.getmtime(obj)
    return m < os.path.getmtime(src) or m < hdr_mtime


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"command failed ({r.returncode}): {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout, r.stderr, flush=True)
    return r


def build(verbose: bool = False, ptxas_verbose: bool = False, debug: bool = False) -> str:
    """Compile all kernels for sm_100a and link ``libkda.so``; returns its path.

    ``debug=True`` builds ``libkda_debug.so`` instead (objects under ``_build_debug/``),
    compiled with ``-DKDA_DEBUG``: every kernel checks the indices it derives from the
    call's data and arithmetic against their extents and reports an out-of-range one in
    the status word (KDA_ERR_DEVICE_BOUNDS) instead of making the access."""
    build_dir, lib, flags = (BUILD_DEBUG, LIB_DEBUG, FLAGS + ["-DKDA_DEBUG"]) if debug else \
        (BUILD, LIB, FLAGS)
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr = max([os.path.getmtime(h) for h in _headers()] + [0.0])
    extra = ["-Xptxas", "-v"] if ptxas_verbose else []
    jobs = []
    objs = []
    for src in srcs:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if ptxas_verbose or _stale(obj, src, hdr):
            jobs.append([NVCC, *ARCH, *flags, *extra, "-c", src, "-o", obj])
    if jobs:
        with ThreadPoolExecutor(max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
            results = list(ex.map(lambda c: _run(c, verbose), jobs))
        if ptxas_verbose:
            for r in results:
                print(r.stderr)
    if jobs or not os.path.exists(lib):
        _run([NVCC, *ARCH, "-shared", "-o", lib, *objs], verbose)
    return lib


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, ptxas_verbose="--ptxas" in sys.argv,
                debug="--debug" in sys.argv))

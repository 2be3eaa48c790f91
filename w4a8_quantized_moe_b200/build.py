"""Build the CUDA library ``libw4a8.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m w4a8_quantized_moe_b200.build [--force] [--verbose]
[--debug-bounds]``.  Objects go to ``w4a8_quantized_moe_b200/_build/``; the
shared library is written next to this file so that it ships with the source
tree.

``--debug-bounds`` builds ``libw4a8_debug.so`` instead (objects in
``_build_debug/``): the same kernels with every routing-derived index checked
against its buffer before use (``W4A8_DEBUG_BOUNDS=1``); an index out of range
raises the device latch's index bit, which ``w4a8_check_device_error`` reports
as ``W4A8_ERR_DEVICE_INDEX``, and the access is skipped.  The binding loads it
when ``W4A8_LIBRARY=debug``.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libw4a8.so")
BUILD_DEBUG = os.path.join(PKG, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "libw4a8_debug.so")
SOURCES = ["kernels_small.cu", "grouped_gemm.cu", "capi.cu", "route_static.cu"]
HEADERS = ["internal.h", "ptx.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = [os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"]
    for c in cand:
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found (set NVCC or put CUDA's bin on PATH)")


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "w4a8.h"))
    files.append(os.path.abspath(__file__))
    return files


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _inputs())


def _compile(src: str, verbose: bool, debug: bool = False) -> str:
    obj = os.path.join(BUILD_DEBUG if debug else BUILD, os.path.basename(src).replace(".cu", ".o"))
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include"),
           "-c", src, "-o", obj]
    if debug:
        cmd.insert(1, "-DW4A8_DEBUG_BOUNDS=1")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, debug_bounds: bool = False) -> str:
    """Compile every source for sm_100a and link ``libw4a8.so`` (or, with
    ``debug_bounds``, ``libw4a8_debug.so``); returns its path."""
    lib = LIB_DEBUG if debug_bounds else LIB
    if not force and not is_stale(lib):
        return lib
    os.makedirs(BUILD_DEBUG if debug_bounds else BUILD, exist_ok=True)
    srcs = [os.path.join(CSRC, f) for f in SOURCES]
    with cf.ThreadPoolExecutor(max_workers=len(srcs)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, debug_bounds), srcs))
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, debug_bounds=a.debug_bounds))

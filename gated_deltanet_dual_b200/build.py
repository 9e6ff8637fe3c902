"""Build the in-tree CUDA library libgdn_dual.so for sm_100a with nvcc.

Every .cu file is compiled to an object of its own (in parallel, under _build/ next to the
package), then the objects are linked into one shared library.

The range-checking variant libgdn_dual_debug.so recompiles the files with device-side index
checks (DEBUG_SOURCES) with -DGDN_DEBUG_BOUNDS, and links them with the other objects: a failed
check reports GDN_ERR_BOUNDS instead of touching memory outside its tensor.

Usage: python -m gated_deltanet_dual_b200.build [--force] [--verbose-ptxas] [--debug-bounds]
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libgdn_dual.so")
DEBUG_LIB = os.path.join(PKG, "libgdn_dual_debug.so")
DEBUG_OBJ = os.path.join(OBJ, "debug_bounds")
DEBUG_SOURCES = ("gdn_chunked.cu", "gdn_conv.cu")      # the files with GDN_IN_RANGE checks
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


def deps():
    return sources() + headers()


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in deps())


def _object(src: str, debug: bool = False) -> str:
    return os.path.join(DEBUG_OBJ if debug else OBJ, os.path.basename(src)[:-3] + ".o")


def _compile(src: str, force: bool, verbose_ptxas: bool, debug: bool = False) -> str:
    obj = _object(src, debug)
    newest_dep = max(os.path.getmtime(f) for f in [src] + headers())
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= newest_dep:
        return obj
    tmp = obj + f".tmp{os.getpid()}"
    cmd = ([NVCC] + (["-Xptxas=-v"] if verbose_ptxas else []) + FLAGS + (["-DGDN_DEBUG_BOUNDS"] if debug else [])
           + ["-c", "-o", tmp, src])
    subprocess.check_call(cmd)
    os.replace(tmp, obj)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    os.makedirs(OBJ, exist_ok=True)
    srcs = sources()
    with ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, verbose_ptxas), srcs))
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp] + objs)
    os.replace(tmp, LIB)
    return LIB


def build_debug(force: bool = False) -> str:
    """libgdn_dual_debug.so: the library with the range-checking build of DEBUG_SOURCES."""
    build(force=False)
    if not force and os.path.exists(DEBUG_LIB) and os.path.getmtime(DEBUG_LIB) >= max(os.path.getmtime(f) for f in deps()):
        return DEBUG_LIB
    os.makedirs(DEBUG_OBJ, exist_ok=True)
    srcs = sources()
    dbg = [s for s in srcs if os.path.basename(s) in DEBUG_SOURCES]
    with ThreadPoolExecutor(max_workers=max(1, len(dbg))) as ex:
        dobjs = dict(zip(dbg, ex.map(lambda s: _compile(s, force, False, debug=True), dbg)))
    objs = [dobjs.get(s, _object(s)) for s in srcs]
    tmp = DEBUG_LIB + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp] + objs)
    os.replace(tmp, DEBUG_LIB)
    return DEBUG_LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true", help="also build libgdn_dual_debug.so")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))
    if a.debug_bounds:
        print(build_debug(force=a.force))
    sys.exit(0)

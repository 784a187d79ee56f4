"""Build libsvdq.so (sm_100a) in-tree with nvcc.

    python -m bit_w4a4_quantized_group_b200.build [--verbose] [--debug]

Each source under ``csrc/`` is compiled to an object in ``_build/`` (in
parallel), then linked into ``_lib/libsvdq.so`` with the CUDA runtime linked
statically.  No GPU is needed to build.

``--debug`` builds ``_lib/libsvdq_debug.so`` instead (objects in ``_build_debug/``):
the same kernels compiled with -DSVDQ_DEBUG, in which every plain global or
shared-memory access of the kernels checks its index first; an access that
would fall outside its buffer is skipped and recorded in the device error word
(sites 201 and 202 of svdq_get_last_device_error).
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIBDIR = os.path.join(PKG, "_lib")
LIB = os.path.join(LIBDIR, "libsvdq.so")
BUILD_DEBUG = os.path.join(PKG, "_build_debug")
LIB_DEBUG = os.path.join(LIBDIR, "libsvdq_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def _sources():
    srcs = []
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cpp")):
            srcs.append(os.path.join(CSRC, f))
    return srcs


def _deps_mtime():
    m = 0.0
    for d in (CSRC, INCLUDE):
        for f in os.listdir(d):
            m = max(m, os.path.getmtime(os.path.join(d, f)))
    return m


def _compile(src: str, verbose: bool, debug: bool = False) -> str:
    obj = os.path.join(BUILD_DEBUG if debug else BUILD, os.path.basename(src) + ".o")
    cmd = [nvcc(), *ARCH, *COMMON, *(["-DSVDQ_DEBUG"] if debug else []), "-c", src, "-o", obj]
    if src.endswith(".cu"):
        cmd += ["-lineinfo"]
        if verbose:
            cmd += ["-Xptxas", "-v"]
    else:
        cmd += ["-x", "c++"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every CUDA / C++ source of the library for sm_100a; return the .so path
    (the bounds-checking debug library when debug is true)."""
    lib = LIB_DEBUG if debug else LIB
    if (not force and os.path.exists(lib) and os.path.getmtime(lib) >= _deps_mtime()):
        return lib
    os.makedirs(BUILD_DEBUG if debug else BUILD, exist_ok=True)
    os.makedirs(LIBDIR, exist_ok=True)
    srcs = _sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, debug), srcs))
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))

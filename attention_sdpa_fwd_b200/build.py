"""Build libsdpa.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m attention_sdpa_fwd_b200.build [--force] [--verbose] [--debug]

Each CUDA source compiles to its own object in parallel (``_build/``), then
one nvcc link makes the shared library.  ``--debug`` builds
``libsdpa_debug.so`` with ``-DSDPA_DEBUG``: the same kernels with their
device-side index checks compiled in (see ``sdpa_debug_checks`` in
``include/sdpa.h``).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsdpa.so")
DEBUG_LIB = os.path.join(PKG, "libsdpa_debug.so")
OBJ_ROOT = os.path.join(PKG, "_build")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsdpa")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def lib_path(debug: bool = False) -> str:
    return DEBUG_LIB if debug else LIB


def needs_build(debug: bool = False) -> bool:
    out = lib_path(debug)
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    out = lib_path(debug)
    if not force and not needs_build(debug):
        return out
    objdir = os.path.join(OBJ_ROOT, "debug" if debug else "release")
    os.makedirs(objdir, exist_ok=True)
    extra = ["-DSDPA_DEBUG"] if debug else []
    if verbose:
        extra.append("-Xptxas=-v")

    def compile_one(src: str) -> str:
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc(), *NVCC_FLAGS, *ARCH_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        return obj

    srcs = sources()
    with ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = out + ".tmp"
    subprocess.run([nvcc(), "-shared", *ARCH_FLAGS, *objs, "-o", tmp], check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))

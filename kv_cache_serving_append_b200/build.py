"""Build librtv.so in-tree with nvcc for sm_100a (no GPU needed to compile).

    python -m kv_cache_serving_append_b200.build [--force] [--debug]

--debug builds librtv_debug.so instead: the same library compiled with
RTV_DEBUG, whose kernels bounds-check the slot indices they are given and
report a violation through the error word (rtv_poll_error -> RTV_ERR_BOUNDS).
The binding loads it when RTV_LIBRARY=debug is set.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "librtv.so")
LIB_DEBUG = os.path.join(HERE, "librtv_debug.so")   # RTV_DEBUG: kernels bounds-check slot indices
SOURCES = ["rtv_cache.cu", "append_kernel.cu", "attend_kernel.cu", "project_kernel.cu"]
HEADERS = ["rtv_internal.h", "sm100.cuh", os.path.join("..", "..", "include", "rtv.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [__file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug: bool = False) -> str:
    """Compile librtv.so (or, with debug, librtv_debug.so with RTV_DEBUG)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    objdir = os.path.join(HERE, "_build", "debug" if debug else "release")
    os.makedirs(objdir, exist_ok=True)
    flags = [*NVCC_FLAGS, *extra_flags] + (["-DRTV_DEBUG"] if debug else [])
    objs = []
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        cmd = [_nvcc(), *flags, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [_nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp, *objs,
           "-lcudart"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv,
          extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])

"""Build the two native libraries of the package, in-tree.

- ``libpa.so``: the CUDA C-ABI library (include/pa.h), compiled by nvcc for
  sm_100a only, with the CUDA runtime linked statically.
- ``libpa_pool.so``: the host block pool (include/pa_pool.h), plain C++17.

Run as ``python paged_kv_cache_333_b200/build.py``.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBPA = os.path.join(PKG, "libpa.so")
LIBPOOL = os.path.join(PKG, "libpa_pool.so")

CUDA_SOURCES = ["pa_lib.cu"]
CUDA_DEPS = ["pa_lib.cu", "attend.cuh", "attend_tc.cuh", "decode.cuh", "decode_mma.cuh", "decode_fp8.cuh", "kv_ops.cuh", "pa_device.cuh"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared",
              "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build_cuda(force: bool = False, verbose: bool = False) -> str:
    deps = [os.path.join(CSRC, f) for f in CUDA_DEPS] + [os.path.join(INCLUDE, "pa.h")]
    if force or _stale(LIBPA, deps):
        cmd = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-o", LIBPA + ".tmp",
               *[os.path.join(CSRC, f) for f in CUDA_SOURCES]]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.check_call(cmd)
        os.replace(LIBPA + ".tmp", LIBPA)
    return LIBPA


def build_pool(force: bool = False) -> str:
    src = os.path.join(CSRC, "pool.cpp")
    if force or _stale(LIBPOOL, [src, os.path.join(INCLUDE, "pa_pool.h")]):
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-Wall", "-Wextra",
                               "-I", INCLUDE, "-o", LIBPOOL + ".tmp", src])
        os.replace(LIBPOOL + ".tmp", LIBPOOL)
    return LIBPOOL


def build_all(force: bool = False, verbose: bool = False) -> None:
    build_pool(force)
    build_cuda(force, verbose)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv, verbose="-v" in sys.argv)

"""Build the MC-Sparse CUDA libraries (libmcs.so, libmcs_micro.so) in-tree for sm_100a."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG_DIR, "csrc")
LIB_PATH = os.path.join(PKG_DIR, "libmcs.so")
MICRO_LIB_PATH = os.path.join(PKG_DIR, "libmcs_micro.so")
SOURCES = ["mcs_api.cu"]
MICRO_SOURCES = ["micro_gather.cu", "micro_pipes.cu"]
HEADERS = ["mcs_common.cuh", "ablation_kernels.cuh", "attn_kernel.cuh", "attn_dual_kernel.cuh", "pair_kernel.cuh", "colsum_kernel.cuh", "topk_kernel.cuh",
           "group_kernels.cuh", "validate_kernels.cuh", "residual_compact.cuh"]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs(sources, header):
    root = os.path.dirname(PKG_DIR)
    files = [os.path.join(CSRC, f) for f in sources + HEADERS]
    files.append(os.path.join(root, "include", "mcs.h"))
    files.append(os.path.join(root, "include", header))
    files.append(os.path.abspath(__file__))
    return files


def _up_to_date(lib, sources, header) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs(sources, header) if os.path.exists(f))


def up_to_date() -> bool:
    return (_up_to_date(LIB_PATH, SOURCES, "mcs.h")
            and _up_to_date(MICRO_LIB_PATH, MICRO_SOURCES, "mcs_micro.h"))


def _compile(lib, sources, verbose):
    tmp = lib + ".tmp"
    cmd = [_nvcc(), *NVCC_FLAGS, "-o", tmp] + [os.path.join(CSRC, s) for s in sources]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libmcs.so (the hot path) and libmcs_micro.so (the gather, MMA
    and exponential microbenchmarks) in-tree for sm_100a; returns libmcs.so's
    path."""
    if force or not _up_to_date(LIB_PATH, SOURCES, "mcs.h"):
        _compile(LIB_PATH, SOURCES, verbose)
    if force or not _up_to_date(MICRO_LIB_PATH, MICRO_SOURCES, "mcs_micro.h"):
        _compile(MICRO_LIB_PATH, MICRO_SOURCES, verbose)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))

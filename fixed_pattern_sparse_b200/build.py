"""Build libskiparse.so (the C-ABI library with the sm_100a kernels) in-tree with nvcc, and
its debug build libskiparse_debug.so (SKIPARSE_DEBUG=1: every token row a kernel computes is
checked against its tensor; see skiparse_debug_shrink_bounds in include/skiparse.h).

    python -m fixed_pattern_sparse_b200.build [--force] [--verbose] [--debug]

nvcc cross-compiles for sm_100a without a GPU. The library links the CUDA runtime
statically and reaches the driver's tensor-map encoder through cudaGetDriverEntryPoint,
so it needs no libcuda at link time.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libskiparse.so")
DEBUG_LIB = os.path.join(HERE, "libskiparse_debug.so")
SOURCES = ["skiparse_api.cu", "attn_fwd_sm100.cu", "attn_bwd_sm100.cu", "rearrange.cu", "no_alloc.cu",
           "host_pipeline.cu", "diag_sm100.cu"]
HEADERS = ["ptx_sm100.cuh", "skiparse_internal.cuh", "attn_common.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _deps():
    return ([os.path.join(CSRC, s) for s in SOURCES + HEADERS]
            + [os.path.join(INCLUDE, "skiparse.h"), os.path.abspath(__file__)])


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and os.path.exists(lib):
        if os.path.getmtime(lib) >= max(os.path.getmtime(p) for p in _deps()):
            return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
           "-I", INCLUDE, "-o", tmp] + [os.path.join(CSRC, s) for s in SOURCES]
    if debug:
        cmd.insert(1, "-DSKIPARSE_DEBUG=1")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))

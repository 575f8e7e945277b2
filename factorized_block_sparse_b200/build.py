"""Builds the in-tree shared library ``libsparse_attn.so`` for sm_100a.

One nvcc invocation compiles the CUDA translation unit (kernels and C ABI)
and the host layout builder.  The CUDA runtime is linked statically and the
driver is reached through ``cudaGetDriverEntryPoint``, so the library loads
on a host without a GPU (for the CPU tests of the layout builder and the
exported symbols) and needs only the NVIDIA driver on a GPU host.
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libsparse_attn.so")
# The failure-detection tests' build: short device-side wait limits, a flag
# that withholds one load, range checks of the device tables, and two
# exported test hooks.  Never used by the product path.
TEST_LIB = os.path.join(HERE, "libsparse_attn_test.so")
SOURCES = [os.path.join(HERE, "csrc", "sa_api.cu"), os.path.join(HERE, "csrc", "sa_layout.cpp")]
HEADERS = [os.path.join(ROOT, "include", "sparse_attn.h")] + [
    os.path.join(HERE, "csrc", f) for f in ("sa_internal.h", "sa_device.cuh", "sa_fwd.cuh", "sa_bwd.cuh",
                                            "sa_tail.cuh")]


def nvcc_path():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def command(out=LIB, extra=()):
    return [nvcc_path(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
            "-lineinfo", "-Xcompiler", "-fPIC,-O3", "-shared", "-cudart", "static",
            "-Xlinker", "-soname=" + os.path.basename(out),
            "-I", os.path.join(ROOT, "include"), "-o", out, *extra, *SOURCES]


def up_to_date(out=LIB):
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(p) <= t for p in SOURCES + HEADERS)


def build(force=False, verbose=False, extra=()):
    """Compile the library if any source is newer than it; return its path."""
    if not force and up_to_date():
        return LIB
    cmd = command(extra=list(extra))
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return LIB


def build_test_lib(force=False, verbose=False):
    """Compile the test build (-DSA_TEST_HOOKS) if it is out of date; return its path."""
    if not force and up_to_date(TEST_LIB):
        return TEST_LIB
    cmd = command(out=TEST_LIB, extra=["-DSA_TEST_HOOKS"])
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return TEST_LIB


# The Sparse Transformer block around the op: its own library, linked against
# libsparse_attn.so (found next to it) and cuBLAS (the projections).
BLOCK_LIB = os.path.join(HERE, "libsparse_block.so")
BLOCK_SOURCES = [os.path.join(HERE, "csrc", "sb_block.cu")]
BLOCK_HEADERS = [os.path.join(ROOT, "include", "sparse_block.h"), os.path.join(ROOT, "include", "sparse_attn.h")]


def cuda_lib_dir():
    return os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "lib64")


def build_block_lib(force=False, verbose=False):
    """Compile libsparse_block.so (after libsparse_attn.so) if out of date; return its path."""
    build()
    if not force and os.path.exists(BLOCK_LIB):
        t = os.path.getmtime(BLOCK_LIB)
        if all(os.path.getmtime(p) <= t for p in BLOCK_SOURCES + BLOCK_HEADERS + [LIB]):
            return BLOCK_LIB
    cmd = [nvcc_path(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-Xcompiler", "-fPIC,-O3", "-shared", "-cudart", "static", "-Xlinker", "-soname=libsparse_block.so",
           "-I", os.path.join(ROOT, "include"), "-o", BLOCK_LIB, *BLOCK_SOURCES,
           "-L", HERE, "-lsparse_attn", "-L", cuda_lib_dir(), "-lcublas", "-lcublasLt",
           "-Xlinker", "-rpath,$ORIGIN", "-Xlinker", "-rpath," + cuda_lib_dir()]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return BLOCK_LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
    build_test_lib(force="--force" in sys.argv, verbose=True)
    build_block_lib(force="--force" in sys.argv, verbose=True)

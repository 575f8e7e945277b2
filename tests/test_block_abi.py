"""C ABI of the block library on the host (no GPU): it loads next to the
attention library, exports every function include/sparse_block.h declares,
links the CUDA runtime statically, and sizes its workspace (0 for shapes it
refuses)."""

import ctypes
import os
import re
import subprocess

import pytest

from factorized_block_sparse_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sb():
    build.build_block_lib()
    from factorized_block_sparse_b200 import sparse_block

    return sparse_block


def test_every_declared_block_function_is_exported(sb):
    text = open(os.path.join(ROOT, "include", "sparse_block.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    declared = set(re.findall(r"\b(sparse_block_\w+)\s*\(", text))
    assert declared == set(sb.EXPORTS)
    raw = ctypes.CDLL(sb.LIB_PATH)
    for name in declared:
        assert hasattr(raw, name), name


def test_block_library_links(sb):
    out = subprocess.run(["ldd", sb.LIB_PATH], capture_output=True, text=True).stdout
    assert "libsparse_attn.so" in out and "libcublas" in out
    assert "libcudart.so" not in out and "libcuda.so" not in out


def test_block_workspace_size(sb):
    from factorized_block_sparse_b200 import sparse_attn as sa

    lay = sa.Layout("fixed", 1024, 128, 32, 64)
    ws = sb.lib.sparse_block_workspace_size
    n = ws(2, 1024, 4, 64, lay.handle)
    mc = 2 * 1024 * 4 * 64 * 2  # one [M, C] bf16 tensor
    # activations of the recomputed forward and their gradients (38 [M, C] tensors) + the attention's workspace
    assert n >= 38 * mc + sa.sparse_attn_bwd_workspace_size(2, 4, 1024, 64, lay)
    assert ws(2, 1024, 4, 48, lay.handle) == 0        # D outside {32, 64, 128}
    assert ws(1, 1024, 64, 128, lay.handle) == 0      # H * D above 6144
    assert ws(0, 1024, 4, 64, lay.handle) == 0
    assert ws(1, 1024, 4, 64, None) == 0


def test_gelu_argument_checks(sb):
    # refused before anything reaches the device (no GPU needed)
    from factorized_block_sparse_b200 import sparse_attn as sa

    f = sb.lib.sparse_block_gelu
    a, b, c = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000)
    assert f(None, b, None, 8, None) == sa.SA_ERR_INVALID_ARG           # u null
    assert f(a, None, None, 8, None) == sa.SA_ERR_INVALID_ARG           # g null
    assert f(a, b, None, 12, None) == sa.SA_ERR_INVALID_ARG             # n not a multiple of 8
    assert f(ctypes.c_void_p(0x10008), b, None, 8, None) == sa.SA_ERR_INVALID_ARG  # u not 16-byte aligned
    assert f(a, b, ctypes.c_void_p(0x30004), 8, None) == sa.SA_ERR_INVALID_ARG     # dgelu not aligned
    assert f(a, b, a, 8, None) == sa.SA_ERR_INVALID_ARG                 # dgelu is u
    assert f(a, b, b, 8, None) == sa.SA_ERR_INVALID_ARG                 # dgelu is g
    assert f(a, b, c, 0, None) == sa.SA_OK                              # nothing to do

"""Thin Python binding of the C ABI in ``include/sparse_block.h``: the Sparse
Transformer block around the attention op.

Argument marshalling only: the block runs in ``libsparse_block.so`` (CUDA
kernels for the layer norms, GELU and head layout, cuBLAS and cuBLASLt for
the projections, ``libsparse_attn.so`` for the attention).  Tensors are
``torch.Tensor`` objects on a CUDA device: activations bf16 ``[B, N, C]``
with ``C = H * D``, projection weights bf16 ``[in, out]``, layer-norm
parameters and parameter gradients float32.  There is no CPU fallback.
"""

import ctypes
import os

from . import sparse_attn as sa

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsparse_block.so")

PARAMS = ("ln1_g", "ln1_b", "w_qkv", "w_o", "ln2_g", "ln2_b", "w_1", "w_2")
EXPORTS = ("sparse_block_workspace_size", "sparse_block_fwd", "sparse_block_bwd", "sparse_block_gelu")


class _Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in PARAMS]


def load_library(path=None):
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m factorized_block_sparse_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    I, VP, SZ = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    P = ctypes.POINTER(_Params)
    lib.sparse_block_workspace_size.argtypes = [I, I, I, I, VP]
    lib.sparse_block_workspace_size.restype = SZ
    lib.sparse_block_fwd.argtypes = [VP, P, VP, I, I, I, I, VP, VP, SZ, VP]
    lib.sparse_block_fwd.restype = I
    lib.sparse_block_bwd.argtypes = [VP, VP, P, VP, P, I, I, I, I, VP, VP, SZ, VP]
    lib.sparse_block_bwd.restype = I
    lib.sparse_block_gelu.argtypes = [VP, VP, VP, SZ, VP]
    lib.sparse_block_gelu.restype = I
    return lib


lib = load_library()


def _struct(d):
    return _Params(*[ctypes.c_void_p(d[n].data_ptr()) for n in PARAMS])


def _dims(x, H):
    B, N, C = (int(s) for s in x.shape)
    if C % H:
        raise ValueError("C must be a multiple of H")
    return B, N, C // H


def workspace(B, N, H, D, layout, device):
    import torch

    n = int(lib.sparse_block_workspace_size(B, N, H, D, layout.handle))
    if n == 0:
        raise sa.SparseAttnError(sa.SA_ERR_INVALID_ARG, "sparse_block_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def sparse_block_fwd(x, params, y, H, layout, ws, stream=None):
    B, N, D = _dims(x, H)
    p = _struct(params)
    sa._check(lib.sparse_block_fwd(sa._ptr(x), ctypes.byref(p), sa._ptr(y), B, N, H, D, layout.handle, sa._ptr(ws),
                                   ws.numel(), sa._stream_ptr(stream)), "sparse_block_fwd")


def sparse_block_bwd(x, dy, params, dx, grads, H, layout, ws, stream=None):
    B, N, D = _dims(x, H)
    p, g = _struct(params), _struct(grads)
    sa._check(lib.sparse_block_bwd(sa._ptr(x), sa._ptr(dy), ctypes.byref(p), sa._ptr(dx), ctypes.byref(g), B, N, H,
                                   D, layout.handle, sa._ptr(ws), ws.numel(), sa._stream_ptr(stream)),
              "sparse_block_bwd")


def forward(x, params, H, layout, ws=None, stream=None):
    """Allocates ``y`` (and a workspace if none is given) and runs the block."""
    import torch

    B, N, D = _dims(x, H)
    ws = workspace(B, N, H, D, layout, x.device) if ws is None else ws
    y = torch.empty_like(x)
    sparse_block_fwd(x, params, y, H, layout, ws, stream)
    return y


def backward(x, dy, params, H, layout, ws=None, stream=None):
    """``(dx, grads)``: grads holds float32 tensors of the parameters' shapes."""
    import torch

    B, N, D = _dims(x, H)
    ws = workspace(B, N, H, D, layout, x.device) if ws is None else ws
    dx = torch.empty_like(x)
    grads = {n: torch.empty(params[n].shape, dtype=torch.float32, device=x.device) for n in PARAMS}
    sparse_block_bwd(x, dy, params, dx, grads, H, layout, ws, stream)
    return dx, grads


def sparse_block_gelu(u, g, dgelu=None, stream=None):
    sa._check(lib.sparse_block_gelu(sa._ptr(u), sa._ptr(g), sa._ptr(dgelu) if dgelu is not None else None,
                                    u.numel(), sa._stream_ptr(stream)), "sparse_block_gelu")


def gelu(u, grad=False, stream=None):
    """``gelu(u)`` (and ``gelu'(u)`` when ``grad``) of a bf16 tensor with a multiple of 8 elements."""
    import torch

    g = torch.empty_like(u)
    d = torch.empty_like(u) if grad else None
    sparse_block_gelu(u, g, d, stream)
    return (g, d) if grad else g

"""Thin Python binding of the C ABI in ``include/sparse_attn.h``.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libsparse_attn.so``.  Tensors are ``torch.Tensor`` objects on a
CUDA device (bf16 ``[B, H, N, D]`` contiguous; lse fp32 ``[B, H, N]``); the
stream is torch's current stream unless one is given.  There is no CPU
fallback: if the library is missing, loading this module raises.
"""

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsparse_attn.so")

PATTERNS = {"all": 0, "local": 1, "strided": 2, "fixed": 3, "column": 4, "block": 5,
            "blocks": 6}  # "blocks": a caller's block mask (Layout.from_blocks)
VIEWS = {"N": 0, "T": 1, "S": 2}
VIEW_TRANSPOSED = 4
SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_CUDA, SA_ERR_LUT, SA_ERR_TIMEOUT, SA_ERR_WORKSPACE = range(7)

# Every entry point declared in include/sparse_attn.h.
EXPORTS = (
    "sparse_attn_layout", "sparse_attn_layout_blocks", "sparse_attn_layout_export", "sparse_attn_layout_info",
    "sparse_attn_layout_upload", "sparse_attn_layout_free", "sparse_attn_fwd", "sparse_attn_fwd_ex",
    "sparse_attn_bwd_workspace_size", "sparse_attn_bwd", "sparse_attn_bwd_ex", "sparse_attn_bwd_noalloc",
    "sparse_attn_status",
    "sparse_attn_strerror", "sparse_attn_kernel_kinds", "sparse_attn_timing_enable",
    "sparse_attn_timing_reset", "sparse_attn_timing_read", "sparse_attn_launch_count",
)


class SparseAttnError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {strerror(status)} (status {status})")


def load_library(path=None):
    """ctypes handle of the library at ``path`` (default: the product build)
    with the argument types of every entry point set."""
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m factorized_block_sparse_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    P, I, F, VP = ctypes.POINTER, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
    lib.sparse_attn_layout.argtypes = [I, I, I, I, I, P(VP)]
    lib.sparse_attn_layout.restype = I
    lib.sparse_attn_layout_blocks.argtypes = [I, I, VP, VP, P(VP)]
    lib.sparse_attn_layout_blocks.restype = I
    lib.sparse_attn_layout_export.argtypes = [VP, I, VP, VP, VP, P(I), P(I)]
    lib.sparse_attn_layout_export.restype = I
    lib.sparse_attn_layout_info.argtypes = [VP, P(I), P(I), P(I), P(I), P(I)]
    lib.sparse_attn_layout_info.restype = I
    lib.sparse_attn_layout_upload.argtypes = [VP, VP]
    lib.sparse_attn_layout_upload.restype = I
    lib.sparse_attn_layout_free.argtypes = [VP]
    lib.sparse_attn_layout_free.restype = None
    lib.sparse_attn_fwd.argtypes = [VP, VP, VP, VP, VP, I, I, I, I, VP, VP]
    lib.sparse_attn_fwd.restype = I
    lib.sparse_attn_fwd_ex.argtypes = [VP, VP, VP, VP, VP, I, I, I, I, ctypes.c_float, VP, VP]
    lib.sparse_attn_fwd_ex.restype = I
    lib.sparse_attn_bwd_workspace_size.argtypes = [I, I, I, I, VP]
    lib.sparse_attn_bwd_workspace_size.restype = ctypes.c_size_t
    lib.sparse_attn_bwd.argtypes = [VP] * 9 + [I, I, I, I, VP, VP, ctypes.c_size_t, VP]
    lib.sparse_attn_bwd.restype = I
    lib.sparse_attn_bwd_ex.argtypes = [VP] * 9 + [I, I, I, I, ctypes.c_float, VP, VP, ctypes.c_size_t, VP]
    lib.sparse_attn_bwd_ex.restype = I
    lib.sparse_attn_bwd_noalloc.argtypes = [VP] * 9 + [I, I, I, I, VP, VP]
    lib.sparse_attn_bwd_noalloc.restype = I
    lib.sparse_attn_status.argtypes = [VP]
    lib.sparse_attn_status.restype = I
    lib.sparse_attn_strerror.argtypes = [I]
    lib.sparse_attn_strerror.restype = ctypes.c_char_p
    lib.sparse_attn_kernel_kinds.argtypes = []
    lib.sparse_attn_kernel_kinds.restype = I
    lib.sparse_attn_timing_enable.argtypes = [I]
    lib.sparse_attn_timing_enable.restype = I
    lib.sparse_attn_timing_reset.argtypes = []
    lib.sparse_attn_timing_reset.restype = I
    lib.sparse_attn_timing_read.argtypes = [I, P(ctypes.c_char_p), P(ctypes.c_double), P(ctypes.c_longlong)]
    lib.sparse_attn_timing_read.restype = I
    lib.sparse_attn_launch_count.argtypes = []
    lib.sparse_attn_launch_count.restype = ctypes.c_longlong
    del F
    return lib


lib = load_library()


def strerror(status):
    return lib.sparse_attn_strerror(int(status)).decode()


def _check(status, what):
    if status != SA_OK:
        raise SparseAttnError(status, what)


class Layout:
    """Owns an ``sa_layout*`` built by ``sparse_attn_layout``."""

    def __init__(self, pattern, N, l=1, c=0, block=64):
        self.pattern = pattern
        self.N, self.l, self.c, self.block = int(N), int(l), int(c), int(block)
        h = ctypes.c_void_p()
        _check(lib.sparse_attn_layout(PATTERNS[pattern], self.N, self.l, self.c, self.block,
                                      ctypes.byref(h)), "sparse_attn_layout")
        self._h = h

    @classmethod
    def from_blocks(cls, N, block, row_ptr, col_idx):
        """Layout of a caller's block mask (``sparse_attn_layout_blocks``): per
        query block, the ascending key blocks at or below the diagonal, the
        diagonal block last; block a multiple of 128."""
        self = cls.__new__(cls)
        self.pattern = "blocks"
        self.N, self.l, self.c, self.block = int(N), 1, 0, int(block)
        rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
        ci = np.ascontiguousarray(col_idx, dtype=np.int32)
        if ci.size == 0:
            ci = np.zeros(1, dtype=np.int32)
        h = ctypes.c_void_p()
        _check(lib.sparse_attn_layout_blocks(self.N, self.block, rp.ctypes.data, ci.ctypes.data, ctypes.byref(h)),
               "sparse_attn_layout_blocks")
        self._h = h
        return self

    @property
    def handle(self):
        return self._h

    def export(self, view, transposed=False):
        """Host copy of one view's block table: dict(row_ptr, col_idx, kind, n_rows)."""
        vid = VIEWS[view] | (VIEW_TRANSPOSED if transposed else 0)
        n_rows, nnz = ctypes.c_int(), ctypes.c_int()
        _check(lib.sparse_attn_layout_export(self._h, vid, None, None, None,
                                             ctypes.byref(n_rows), ctypes.byref(nnz)), "export")
        rp = np.zeros(n_rows.value + 1, np.int32)
        ci = np.zeros(max(nnz.value, 1), np.int32)
        kd = np.zeros(max(nnz.value, 1), np.uint8)
        _check(lib.sparse_attn_layout_export(self._h, vid, rp.ctypes.data, ci.ctypes.data, kd.ctypes.data,
                                             ctypes.byref(n_rows), ctypes.byref(nnz)), "export")
        return dict(row_ptr=rp, col_idx=ci[:nnz.value], kind=kd[:nnz.value], n_rows=n_rows.value)

    def upload(self, stream=None):
        _check(lib.sparse_attn_layout_upload(self._h, _stream_ptr(stream)), "sparse_attn_layout_upload")

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib.sparse_attn_layout_free(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def sparse_attn_layout(pattern, N, l=1, c=0, block=64):
    return Layout(pattern, N, l, c, block)


def _stream_ptr(stream):
    if stream is None:
        import torch

        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _shape(q):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, D]")
    return tuple(int(x) for x in q.shape)


def sparse_attn_fwd(q, k, v, o, lse, layout, stream=None, scale=None):
    """Writes ``o`` and ``lse`` in place (C ABI call); ``scale`` None is 1/sqrt(D)."""
    B, H, N, D = _shape(q)
    if scale is None:
        _check(lib.sparse_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, D,
                                   layout.handle, _stream_ptr(stream)), "sparse_attn_fwd")
    else:
        _check(lib.sparse_attn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, D, float(scale),
                                      layout.handle, _stream_ptr(stream)), "sparse_attn_fwd_ex")


def sparse_attn_bwd_workspace_size(B, H, N, D, layout):
    return int(lib.sparse_attn_bwd_workspace_size(B, H, N, D, layout.handle))


def sparse_attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, layout, workspace, stream=None, scale=None):
    """Writes ``dq``, ``dk``, ``dv`` in place (C ABI call); ``scale`` None is 1/sqrt(D)."""
    B, H, N, D = _shape(q)
    ws_bytes = workspace.numel() * workspace.element_size()
    if scale is None:
        _check(lib.sparse_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                                   _ptr(dk), _ptr(dv), B, H, N, D, layout.handle, _ptr(workspace),
                                   ws_bytes, _stream_ptr(stream)), "sparse_attn_bwd")
    else:
        _check(lib.sparse_attn_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                                      _ptr(dk), _ptr(dv), B, H, N, D, float(scale), layout.handle,
                                      _ptr(workspace), ws_bytes, _stream_ptr(stream)), "sparse_attn_bwd_ex")


def sparse_attn_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, layout, stream=None):
    """Backward pass that allocates nothing: it runs in the library's built-in
    scratch array (SA_NOALLOC_SCRATCH_BYTES per device) instead of a caller
    workspace.  For callers that may not allocate device memory.  The layout
    must already be on the device (``layout.upload()``); calls that overlap on
    the GPU share the scratch array and race."""
    B, H, N, D = _shape(q)
    _check(lib.sparse_attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                                       _ptr(dk), _ptr(dv), B, H, N, D, layout.handle, _stream_ptr(stream)),
           "sparse_attn_bwd_noalloc")


NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


def sparse_attn_status(stream=None):
    return int(lib.sparse_attn_status(_stream_ptr(stream)))


# ------------------------------------------------------------ conveniences
def forward(q, k, v, layout, stream=None, scale=None):
    """Allocates ``o`` (bf16) and ``lse`` (fp32) with torch and runs the forward pass."""
    import torch

    B, H, N, D = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    sparse_attn_fwd(q, k, v, o, lse, layout, stream, scale)
    return o, lse


def workspace(B, H, N, D, layout, device):
    import torch

    n = sparse_attn_bwd_workspace_size(B, H, N, D, layout)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def backward(q, k, v, o, lse, dO, layout, ws=None, stream=None, scale=None):
    """Allocates ``dq``, ``dk``, ``dv`` (and a workspace if none is given)."""
    import torch

    B, H, N, D = _shape(q)
    if ws is None:
        ws = workspace(B, H, N, D, layout, q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    sparse_attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, layout, ws, stream, scale)
    return dq, dk, dv


def kernel_times():
    """{kernel name: (total ms, launches)} recorded while timing is enabled."""
    out = {}
    for i in range(lib.sparse_attn_kernel_kinds()):
        name, ms, cnt = ctypes.c_char_p(), ctypes.c_double(), ctypes.c_longlong()
        _check(lib.sparse_attn_timing_read(i, ctypes.byref(name), ctypes.byref(ms), ctypes.byref(cnt)),
               "timing_read")
        out[name.value.decode()] = (ms.value, cnt.value)
    return out


def timing_enable(on=True):
    lib.sparse_attn_timing_enable(1 if on else 0)


def timing_reset():
    lib.sparse_attn_timing_reset()


def launch_count():
    return int(lib.sparse_attn_launch_count())

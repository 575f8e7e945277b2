"""Failure detection on the GPU, without a GPU fault.

The kernels never trap: every device-side wait is bounded, and a wait that
runs out records SA_ERR_TIMEOUT in the device status word, drains what is in
flight and returns; sparse_attn_status() reports it and the process carries
on.  These tests use the library's test build (libsparse_attn_test.so: the
same sources compiled with SA_TEST_HOOKS), whose waits give up after a few
milliseconds and which exports two hooks:

* sparse_attn_test_withhold(1) makes the backward pass's producer skip the
  first load of each CTA, so a consumer's wait runs out (a flag that nothing
  sets);
* sparse_attn_test_corrupt_entry() overwrites one entry of a device tile
  table; the test build range-checks the tables before its kernels run and
  records SA_ERR_LUT, and the kernels then return without touching anything.

Neither case can fault: the withheld load is never issued, and the corrupted
entry (a tile index far past the end) would only address positions that a
tensor-map load fills with zeros.
"""

import ctypes
import time

import numpy as np
import pytest
import torch

from factorized_block_sparse_b200 import build, synth
from gpu_util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tl():
    from factorized_block_sparse_b200 import sparse_attn as sa

    lib = sa.load_library(build.build_test_lib())
    lib.sparse_attn_test_withhold.argtypes = [ctypes.c_int]
    lib.sparse_attn_test_withhold.restype = ctypes.c_int
    lib.sparse_attn_test_corrupt_entry.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int]
    lib.sparse_attn_test_corrupt_entry.restype = ctypes.c_int
    return lib


def _layout(lib, mode, N, l, c, block):
    from factorized_block_sparse_b200 import sparse_attn as sa

    h = ctypes.c_void_p()
    assert lib.sparse_attn_layout(sa.PATTERNS[mode], N, l, c, block, ctypes.byref(h)) == sa.SA_OK
    return h


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_withheld_load_times_out_then_recovers(cuda_device, tl):
    from factorized_block_sparse_b200 import sparse_attn as sa

    # dense causal, D = 64: the backward's tables take the wide-step kernel
    B, H, N, D = 1, 2, 1024, 64
    x = synth.inputs(B, H, N, D)
    q, k, v, dO = (x[n].to(cuda_device) for n in ("q", "k", "v", "dO"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=cuda_device)
    h = _layout(tl, "all", N, 1, 0, 64)
    s = sa._stream_ptr(None)
    assert tl.sparse_attn_fwd(_p(q), _p(k), _p(v), _p(o), _p(lse), B, H, N, D, h, s) == sa.SA_OK
    assert tl.sparse_attn_status(s) == sa.SA_OK
    ws = torch.empty(max(tl.sparse_attn_bwd_workspace_size(B, H, N, D, h), 256), dtype=torch.uint8,
                     device=cuda_device)
    grads = [torch.empty_like(q) for _ in range(3)]

    def bwd():
        return tl.sparse_attn_bwd(_p(q), _p(k), _p(v), _p(o), _p(lse), _p(dO), *map(_p, grads), B, H, N, D, h,
                                  _p(ws), ws.numel(), s)

    assert tl.sparse_attn_test_withhold(1) == sa.SA_OK
    t0 = time.perf_counter()
    assert bwd() == sa.SA_OK  # enqueued; the failure shows in the status word
    st = tl.sparse_attn_status(s)
    elapsed = time.perf_counter() - t0
    assert tl.sparse_attn_test_withhold(0) == sa.SA_OK
    assert st == sa.SA_ERR_TIMEOUT, sa.strerror(st)
    assert elapsed < 2.0, f"the timeout took {elapsed:.2f} s"
    # the status word was cleared by reading it, and the context is usable
    assert tl.sparse_attn_status(s) == sa.SA_OK
    assert bwd() == sa.SA_OK
    assert tl.sparse_attn_status(s) == sa.SA_OK
    got = [t.float().cpu().numpy() for t in grads]
    lay = sa.Layout("all", N, 1, 0, 64)
    ref = [t.float().cpu().numpy() for t in sa.backward(q, k, v, o, lse, dO, lay)]
    torch.cuda.synchronize()
    assert_close("recovered dq", got[0], ref[0])
    assert np.array_equal(got[1], ref[1]) and np.array_equal(got[2], ref[2])
    tl.sparse_attn_layout_free(h)


def test_corrupted_table_is_refused(cuda_device, tl):
    from factorized_block_sparse_b200 import sparse_attn as sa

    B, H, N, D = 1, 1, 1024, 64
    x = synth.inputs(B, H, N, D)
    q, k, v = (x[n].to(cuda_device) for n in ("q", "k", "v"))
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=cuda_device)
    s = sa._stream_ptr(None)
    h = _layout(tl, "fixed", N, 128, 32, 64)
    assert tl.sparse_attn_layout_upload(h, s) == sa.SA_OK
    assert tl.sparse_attn_test_corrupt_entry(h, 0, (1 << 22) << 3) == sa.SA_OK  # a tile far past the end
    assert tl.sparse_attn_fwd(_p(q), _p(k), _p(v), _p(o), _p(lse), B, H, N, D, h, s) == sa.SA_OK
    assert tl.sparse_attn_status(s) == sa.SA_ERR_LUT
    # the kernels returned before touching their outputs
    assert torch.isnan(o).all() and torch.isnan(lse).all()
    tl.sparse_attn_layout_free(h)
    # a sound layout runs normally afterwards
    h = _layout(tl, "fixed", N, 128, 32, 64)
    assert tl.sparse_attn_fwd(_p(q), _p(k), _p(v), _p(o), _p(lse), B, H, N, D, h, s) == sa.SA_OK
    assert tl.sparse_attn_status(s) == sa.SA_OK
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    tl.sparse_attn_layout_free(h)

"""The allocation-free backward entry point, sparse_attn_bwd_noalloc.

Some callers may not allocate device memory at all (a host framework that
owns all device memory through its own pool, or a rule against device
allocation after start-up), so they cannot pass the workspace that
sparse_attn_bwd needs.  sparse_attn_bwd_noalloc runs the same backward pass
in a scratch array built into the library.  This file checks, through the C
ABI, that two calls in a row give the results of the workspace entry point
within the parity tolerance, and that it refuses shapes that do not fit and
layouts that are not on the device yet (refusing rather than allocating).

The file is named to be collected last, so a run that stops at the first
failure has run every other test before it.
"""

import numpy as np
import pytest
import torch

from factorized_block_sparse_b200 import synth
from gpu_util import MAX_ABS, REL_L2, assert_close

pytestmark = pytest.mark.gpu

CASES = [
    # mode, B, H, N, D, l, c, block
    ("strided", 1, 2, 2048, 64, 64, 0, 64),
    ("fixed", 2, 1, 2048, 64, 128, 32, 64),
    ("all", 1, 1, 1024, 128, 1, 0, 64),
]


@pytest.mark.parametrize("mode,B,H,N,D,l,c,block", CASES)
def test_noalloc_backward_matches_workspace_backward(cuda_device, mode, B, H, N, D, l, c, block):
    from factorized_block_sparse_b200 import sparse_attn as sa

    assert sa.sparse_attn_bwd_workspace_size(B, H, N, D, sa.Layout(mode, N, l, c, block)) \
        <= sa.NOALLOC_SCRATCH_BYTES
    x = synth.inputs(B, H, N, D)
    q, k, v, dO = (x[n].to(cuda_device) for n in ("q", "k", "v", "dO"))
    lay = sa.Layout(mode, N, l, c, block)
    lay.upload()
    o, lse = sa.forward(q, k, v, lay)
    ref = sa.backward(q, k, v, o, lse, dO, lay)  # the workspace entry point
    torch.cuda.synchronize()
    ref = [t.float().cpu().numpy() for t in ref]
    for call in range(2):  # the scratch array keeps the previous call's contents
        outs = [torch.full_like(q, float("nan")) for _ in range(3)]
        sa.sparse_attn_bwd_noalloc(q, k, v, o, lse, dO, *outs, lay)
        assert sa.sparse_attn_status() == 0
        got = [t.float().cpu().numpy() for t in outs]
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            assert np.isfinite(g).all(), (call, name)
            assert_close(f"call {call} {name}", g, r, MAX_ABS, REL_L2)
        # dk and dv do not use atomics: identical to the workspace entry point
        assert np.array_equal(got[1], ref[1]) and np.array_equal(got[2], ref[2])


def test_noalloc_after_a_larger_different_call(cuda_device):
    """A larger strided call fills more of the scratch array (column-order lse
    blocks, secondary partials) than a smaller fixed or dense call reads; the
    smaller call must not pick up anything the larger one left behind."""
    from factorized_block_sparse_b200 import sparse_attn as sa

    first = ("strided", 1, 4, 4096, 64, 64, 0, 64)
    for second in (("fixed", 1, 1, 1024, 64, 128, 32, 64), ("all", 1, 1, 640, 32, 1, 0, 64)):
        runs = []
        for mode, B, H, N, D, l, c, block in (first, second):
            x = synth.inputs(B, H, N, D, seed_offset=7)
            q, k, v, dO = (x[n].to(cuda_device) for n in ("q", "k", "v", "dO"))
            lay = sa.Layout(mode, N, l, c, block)
            assert sa.sparse_attn_bwd_workspace_size(B, H, N, D, lay) <= sa.NOALLOC_SCRATCH_BYTES
            lay.upload()
            o, lse = sa.forward(q, k, v, lay)
            outs = [torch.full_like(q, float("nan")) for _ in range(3)]
            sa.sparse_attn_bwd_noalloc(q, k, v, o, lse, dO, *outs, lay)
            assert sa.sparse_attn_status() == 0
            runs.append((q, k, v, o, lse, dO, lay, outs))
        q, k, v, o, lse, dO, lay, outs = runs[1]
        ref = [t.float().cpu().numpy() for t in sa.backward(q, k, v, o, lse, dO, lay)]
        got = [t.float().cpu().numpy() for t in outs]
        assert_close(f"{second[0]} after strided dq", got[0], ref[0], MAX_ABS, REL_L2)
        assert np.array_equal(got[1], ref[1]) and np.array_equal(got[2], ref[2]), second[0]


def test_noalloc_refuses_instead_of_allocating(cuda_device):
    from factorized_block_sparse_b200 import sparse_attn as sa

    t = torch.zeros(16, dtype=torch.bfloat16, device=cuda_device)
    lse = torch.zeros(16, dtype=torch.float32, device=cuda_device)
    p = [sa._ptr(t)] * 4
    # a shape whose workspace exceeds the scratch array: rejected before any device work
    big = sa.Layout("all", 65536, 1, 0, 64)
    assert sa.sparse_attn_bwd_workspace_size(1, 16, 65536, 64, big) > sa.NOALLOC_SCRATCH_BYTES
    st = sa.lib.sparse_attn_bwd_noalloc(p[0], p[0], p[0], p[0], sa._ptr(lse), p[0], p[0], p[0], p[0],
                                        1, 16, 65536, 64, big.handle, sa._stream_ptr(None))
    assert st == sa.SA_ERR_WORKSPACE
    # a layout whose tables are not on this device yet: refused (uploading would allocate)
    fresh = sa.Layout("strided", 1024, 32, 0, 32)
    st = sa.lib.sparse_attn_bwd_noalloc(p[0], p[0], p[0], p[0], sa._ptr(lse), p[0], p[0], p[0], p[0],
                                        1, 1, 1024, 64, fresh.handle, sa._stream_ptr(None))
    assert st == sa.SA_ERR_INVALID_ARG
    torch.cuda.synchronize()

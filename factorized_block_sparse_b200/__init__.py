"""Causal factorized sparse self-attention (Sparse Transformer) on B200.

Modes ``all``, ``local``, ``strided`` and ``fixed``, and the single heads of
the two-head form, ``column`` (the strided column head) and ``block`` (the
fixed own-block head); softmax scale 1/sqrt(D) or given.  Forward and
backward run as hand-written sm_100a CUDA kernels (tcgen05 tensor cores with
TMEM accumulators, TMA loads, warp-specialised pipelines) behind the C ABI
declared in ``include/sparse_attn.h``.

Use::

    import torch
    from factorized_block_sparse_b200 import sparse_attn as sa
    lay = sa.Layout("strided", N=12288, l=192, block=64)   # built once per shape
    o, lse = sa.forward(q, k, v, lay)                        # bf16 [B, H, N, D]
    dq, dk, dv = sa.backward(q, k, v, o, lse, dO, lay)

``python -m factorized_block_sparse_b200.build`` compiles the library in
place (nvcc, sm_100a).

Submodules are imported on demand (``from factorized_block_sparse_b200
import sparse_attn``), so that ``factorized_block_sparse_b200.synth``
(seeded inputs) can be used without loading the shared library.  Any
compute call fails loudly when the library is missing; there is no CPU
fallback.
"""

__all__ = ["sparse_attn", "synth", "build"]

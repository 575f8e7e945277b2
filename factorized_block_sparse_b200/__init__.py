"""Causal factorized sparse self-attention (Sparse Transformer) on B200.

Modes ``all``, ``local``, ``strided`` and ``fixed``; forward and backward
run as hand-written sm_100a CUDA kernels (tcgen05 tensor cores with TMEM
accumulators, TMA loads, warp-specialised pipelines) behind the C ABI
declared in ``include/sparse_attn.h``.

Submodules are imported on demand (``from factorized_block_sparse_b200
import sparse_attn``), so that ``factorized_block_sparse_b200.synth``
(seeded inputs) can be used without loading the shared library.  Any
compute call fails loudly when the library is missing; there is no CPU
fallback.
"""

__all__ = ["sparse_attn", "synth", "build"]

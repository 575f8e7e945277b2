"""Shared helpers of the GPU parity tests: run the library through its C ABI
binding on seeded inputs and compare with the float64 oracle."""

import numpy as np
import torch

from factorized_block_sparse_b200 import synth
from oracle import attention

# Tolerances of outputs and gradients computed from bf16 inputs with fp32
# accumulation against the float64 oracle.
MAX_ABS = 2e-2
REL_L2 = 5e-3


def metrics(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = got - ref
    return float(np.abs(err).max()), float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300))


def assert_close(name, got, ref, max_abs=MAX_ABS, rel_l2=REL_L2):
    ma, rl = metrics(got, ref)
    assert ma <= max_abs and rl <= rel_l2, f"{name}: max-abs {ma:.3e} (<= {max_abs}), rel-L2 {rl:.3e} (<= {rel_l2})"
    return ma, rl


def run_library(mode, B, H, N, D, l, c, block, seed_offset=0, device="cuda:0", scale=None, layout=None):
    """fwd + bwd through the C ABI; returns host inputs and float64 outputs."""
    from factorized_block_sparse_b200 import sparse_attn as sa

    x = synth.inputs(B, H, N, D, seed_offset)
    lay = layout if layout is not None else sa.Layout(mode, N, l, c, block)
    q, k, v, dO = (x[n].to(device) for n in ("q", "k", "v", "dO"))
    o, lse = sa.forward(q, k, v, lay, scale=scale)
    dq, dk, dv = sa.backward(q, k, v, o, lse, dO, lay, scale=scale)
    torch.cuda.synchronize()
    st = sa.sparse_attn_status()
    assert st == 0, f"device status {st}: {sa.strerror(st)}"
    out = {n: t.float().cpu().double().numpy() for n, t in
           (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}
    return x, out, lay


def oracle_full(x, mode, l, c, scale=None):
    q, k, v, dO = (synth.to_f64(x[n]) for n in ("q", "k", "v", "dO"))
    O, L = attention.forward(q, k, v, mode, l, c, scale=scale)
    dq, dk, dv = attention.backward(q, k, v, dO, mode, l, c, scale=scale, lse=L)
    return {"o": O, "lse": L, "dq": dq, "dk": dk, "dv": dv}

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


def bf16_half_spacing(ref):
    """Half the spacing of bfloat16 numbers at |ref| (8 significant bits):
    the distance from an exact value to its nearest bfloat16 can reach this,
    whatever the arithmetic before the final rounding."""
    a = np.abs(np.asarray(ref, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, np.finfo(np.float64).tiny)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def metrics(got, ref, bf16=False):
    """(max-abs error, rel-L2 error, max-abs error beyond the bf16 output rounding)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    beyond = err - bf16_half_spacing(ref) if bf16 else err
    return (float(err.max()), float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)),
            float(beyond.max()))


def assert_close(name, got, ref, max_abs=MAX_ABS, rel_l2=REL_L2, bf16=None):
    """Max-abs and rel-L2 bounds.  For bfloat16 outputs (the default for every
    name but lse) the max-abs bound is taken on top of the output's own
    rounding: |got - ref| <= max_abs + half the bf16 spacing at |ref|.  Below
    |ref| = 1 that adds at most 2^-9; at |ref| in [4, 8) rounding alone can
    reach 2^-6 = 0.0156, most of the plain bound."""
    if bf16 is None:
        bf16 = not name.endswith("lse")
    ma, rl, mb = metrics(got, ref, bf16)
    assert mb <= max_abs and rl <= rel_l2, (
        f"{name}: max-abs {ma:.3e} ({mb:.3e} beyond bf16 rounding; bound {max_abs}), "
        f"rel-L2 {rl:.3e} (<= {rel_l2})")
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


def oracle_full(x, mode, l, c, scale=None, sl=None):
    """The whole oracle forward + backward; ``sl`` = (b, h) restricts it to one slice."""
    q, k, v, dO = (synth.to_f64(x[n]) for n in ("q", "k", "v", "dO"))
    if sl is not None:
        b, h = sl
        q, k, v, dO = (t[b:b + 1, h:h + 1] for t in (q, k, v, dO))
    O, L = attention.forward(q, k, v, mode, l, c, scale=scale)
    dq, dk, dv = attention.backward(q, k, v, dO, mode, l, c, scale=scale, lse=L)
    return {"o": O, "lse": L, "dq": dq, "dk": dk, "dv": dv}

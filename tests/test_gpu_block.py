"""GPU parity of the Sparse Transformer block (libsparse_block.so through its
C ABI) against the float64 block oracle (oracle.block), element by element.

Tolerance.  The block's activations are bf16: on the way to y about ten
intermediates are rounded to bf16 (a, q/k/v, the attention output, h, f, u,
gelu(u), y and the attention's own rounding), each by at most 2^-9 of its
magnitude, and the gradients pass through about twice as many (the
recomputed forward, then dg, gelu'(u), du, df, dh, do, the attention
backward, dqkv, da, dx); the GEMMs accumulate in float32.  Hence the bounds: relative L2
error at most 1e-2 (about sqrt(20) * 2^-9 with room), and every element
within 5e-2 of the largest magnitude of its reference (about 20 * 2^-9),
for y, dx and each parameter gradient.
"""

import numpy as np
import pytest
import torch

from factorized_block_sparse_b200 import synth
from oracle import block as oracle_block

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_REL = 5e-2


def _close(name, got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    rl = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    mr = err.max() / max(np.abs(ref).max(), 1e-300)
    assert np.isfinite(got).all(), name
    assert rl <= REL_L2 and mr <= MAX_REL, f"{name}: rel-L2 {rl:.2e} (<= {REL_L2}), max {mr:.2e} of max|ref| (<= {MAX_REL})"


def _run(mode, B, N, H, D, l, c, block, device):
    from factorized_block_sparse_b200 import sparse_attn as sa
    from factorized_block_sparse_b200 import sparse_block as sb

    C = H * D
    xin = synth.block_inputs(B, N, C)
    p = synth.block_params(C)
    lay = sa.Layout(mode, N, l, c, block)
    x, dy = xin["x"].to(device), xin["dy"].to(device)
    pd = {k: v.to(device) for k, v in p.items()}
    ws = sb.workspace(B, N, H, D, lay, device)
    y = sb.forward(x, pd, H, lay, ws)
    dx, g = sb.backward(x, dy, pd, H, lay, ws)
    torch.cuda.synchronize()
    assert sa.sparse_attn_status() == sa.SA_OK
    got = {"y": y.float().cpu().numpy(), "dx": dx.float().cpu().numpy()}
    got.update({k: v.cpu().numpy() for k, v in g.items()})
    pf = {k: synth.to_f64(v) for k, v in p.items()}
    xf, dyf = synth.to_f64(xin["x"]), synth.to_f64(xin["dy"])
    yr, _ = oracle_block.forward(xf, pf, H, mode, l, c)
    dxr, gr = oracle_block.backward(xf, dyf, pf, H, mode, l, c)
    ref = {"y": yr, "dx": dxr, **gr}
    return got, ref


@pytest.mark.parametrize("mode,B,N,H,D,l,c,block", [
    ("fixed", 1, 512, 2, 64, 128, 32, 64),    # text-like pattern, C = 128
    ("strided", 2, 256, 4, 32, 16, 0, 16),    # tiny-like pattern, C = 128
    ("all", 1, 256, 2, 128, 1, 0, 64),        # D = 128, C = 256
    ("strided", 1, 384, 3, 64, 48, 0, 16),    # C = 192 (not a multiple of 256), R = 8
    # the layer norms' widths: rows in registers with per-lane dg/db sums (C = 512),
    # rows in registers with shared sums (C = 1024), rows read per pass (C = 1536),
    # and shared sums above the default 48 KiB of dynamic shared memory (C = 2048)
    ("fixed", 1, 256, 8, 64, 128, 32, 64),
    ("local", 1, 256, 8, 128, 64, 0, 64),
    ("all", 1, 128, 12, 128, 1, 0, 64),
    ("all", 1, 128, 16, 128, 1, 0, 64),
    # ragged: N = 1000 (M = 2000 rows, no multiple of a tile), a partial last row of the strided view
    ("strided", 2, 1000, 2, 64, 64, 0, 8),
])
def test_block_parity(cuda_device, mode, B, N, H, D, l, c, block):
    got, ref = _run(mode, B, N, H, D, l, c, block, cuda_device)
    for name in ("y", "dx", "ln1_g", "ln1_b", "w_qkv", "w_o", "ln2_g", "ln2_b", "w_1", "w_2"):
        _close(f"{mode} {name}", got[name], ref[name])


def test_block_rejects_bad_arguments(cuda_device):
    from factorized_block_sparse_b200 import sparse_attn as sa
    from factorized_block_sparse_b200 import sparse_block as sb

    H, D, N = 2, 64, 256
    lay = sa.Layout("all", N, 1, 0, 64)
    x = torch.zeros((1, N, H * D), dtype=torch.bfloat16, device=cuda_device)
    p = {k: v.to(cuda_device) for k, v in synth.block_params(H * D).items()}
    ws = sb.workspace(1, N, H, D, lay, cuda_device)
    with pytest.raises(sa.SparseAttnError) as e:
        sb.sparse_block_fwd(x, p, x, H, lay, ws)  # y aliases x
    assert e.value.status == sa.SA_ERR_INVALID_ARG
    with pytest.raises(sa.SparseAttnError) as e:
        sb.sparse_block_fwd(x, p, torch.empty_like(x), H, lay, ws[: ws.numel() // 2])
    assert e.value.status == sa.SA_ERR_WORKSPACE


def test_gelu_against_fp32_reference(cuda_device):
    """The block's GELU and its derivative against PyTorch's exact (erf) GELU
    in float32 and its derivative in float64, on the same bf16 inputs: within
    half a bf16 spacing of the reference (the output's own rounding) plus
    1e-6 (the approximation of Phi, below 7.5e-8 absolute, times |u| <= 12)."""
    from factorized_block_sparse_b200 import sparse_block as sb

    gen = torch.Generator().manual_seed(30)
    grid = torch.linspace(-12.0, 12.0, 24576)
    u = torch.cat([grid, 2.0 * torch.randn(40960, generator=gen)]).to(torch.bfloat16)
    g, d = sb.gelu(u.to(cuda_device), grad=True)
    g_in_place = u.to(cuda_device)
    sb.sparse_block_gelu(g_in_place, g_in_place)
    torch.cuda.synchronize()
    uf = u.double()
    ref_g = torch.nn.functional.gelu(u.float()).double()
    phi = torch.exp(-0.5 * uf * uf) / np.sqrt(2.0 * np.pi)
    ref_d = 0.5 * (1.0 + torch.erf(uf / np.sqrt(2.0))) + uf * phi

    def half_ulp(x):
        ax = x.abs().clamp_min(2.0 ** -126)
        return 2.0 ** (torch.floor(torch.log2(ax)) - 8)

    for name, got, ref in (("gelu", g, ref_g), ("gelu'", d, ref_d), ("gelu in place", g_in_place, ref_g)):
        got = got.double().cpu()
        err = (got - ref).abs()
        bound = half_ulp(ref) + 1e-6
        assert torch.isfinite(got).all(), name
        assert (err <= bound).all(), f"{name}: worst excess {(err - bound).max().item():.3e}"


def test_block_calls_from_two_threads(cuda_device):
    """Two host threads, each with its own stream and workspace, run forward +
    backward of the block at the same time: the results equal those of one
    thread alone, bit for bit where the block is deterministic (y) and within
    float32 reduction-order noise for the gradients."""
    import threading

    from factorized_block_sparse_b200 import sparse_attn as sa
    from factorized_block_sparse_b200 import sparse_block as sb

    B, N, H, D = 1, 512, 2, 64
    lay = sa.Layout("fixed", N, 128, 32, 64)
    lay.upload()
    p = {k: v.to(cuda_device) for k, v in synth.block_params(H * D).items()}
    xin = synth.block_inputs(B, N, H * D)
    x, dy = xin["x"].to(cuda_device), xin["dy"].to(cuda_device)

    def run(stream, out):
        with torch.cuda.stream(stream):
            ws = sb.workspace(B, N, H, D, lay, cuda_device)
            for _ in range(3):
                y = sb.forward(x, p, H, lay, ws, stream.cuda_stream)
                dx, g = sb.backward(x, dy, p, H, lay, ws, stream.cuda_stream)
            stream.synchronize()
            out.update(y=y.float().cpu(), dx=dx.float().cpu(), w_1=g["w_1"].cpu(), ln1_g=g["ln1_g"].cpu())

    ref = {}
    run(torch.cuda.Stream(device=cuda_device), ref)
    outs = [{}, {}]
    threads = [threading.Thread(target=run, args=(torch.cuda.Stream(device=cuda_device), o)) for o in outs]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert sa.sparse_attn_status() == sa.SA_OK
    for o in outs:
        assert torch.equal(o["y"], ref["y"])
        for name in ("dx", "w_1", "ln1_g"):
            assert torch.allclose(o[name], ref[name], rtol=1e-2, atol=1e-3 * ref[name].abs().max().item()), name

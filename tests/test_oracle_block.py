"""Pins of the float64 block oracle (oracle.block) against things other than
itself (CPU only).

* the whole block in torch float64 (layer_norm, exact gelu, matmuls, a
  masked softmax attention built from torch ops) and its gradients by
  autograd: an independent implementation of the same reading;
* central finite differences of sum(y * dy) against the analytic backward;
* closed forms: zero output projections make the block the identity
  (y == x, dx == dy); layer norm of a constant row is its bias; gelu(0) = 0,
  gelu'(0) = 1/2, gelu(u) -> u and gelu'(u) -> 1 for large u.
"""

import numpy as np
import pytest
import torch

from factorized_block_sparse_b200 import synth
from oracle import block, patterns


def _params(C, seed=20):
    return {k: synth.to_f64(v) for k, v in synth.block_params(C, seed).items()}


def _torch_block(x, dy, p, H, mode, l, c):
    """y, dx and parameter gradients by torch autograd (float64)."""
    tp = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in p.items()}
    tx = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    B, N, C = x.shape
    D = C // H
    F = torch.nn.functional
    a = F.layer_norm(tx, (C,), tp["ln1_g"], tp["ln1_b"], eps=1e-5)
    qkv = a @ tp["w_qkv"]
    q, k, v = (qkv[..., i * C:(i + 1) * C].reshape(B, N, H, D).transpose(1, 2) for i in range(3))
    m = torch.tensor(patterns.mask(mode, N, l, c))
    s = (q @ k.transpose(-1, -2)) / np.sqrt(D)
    att = torch.softmax(s.masked_fill(~m, float("-inf")), dim=-1) @ v
    h = tx + att.transpose(1, 2).reshape(B, N, C) @ tp["w_o"]
    f = F.layer_norm(h, (C,), tp["ln2_g"], tp["ln2_b"], eps=1e-5)
    y = h + F.gelu(f @ tp["w_1"], approximate="none") @ tp["w_2"]
    y.backward(torch.tensor(dy, dtype=torch.float64))
    return y.detach().numpy(), tx.grad.numpy(), {k: t.grad.numpy() for k, t in tp.items()}


@pytest.mark.parametrize("mode,B,N,H,D,l,c", [
    ("strided", 1, 64, 2, 8, 8, 0),
    ("fixed", 2, 48, 2, 4, 16, 4),
    ("all", 1, 32, 1, 8, 1, 0),
])
def test_block_matches_torch_autograd(mode, B, N, H, D, l, c):
    C = H * D
    rng = np.random.default_rng(0)
    x = rng.standard_normal((B, N, C))
    dy = rng.standard_normal((B, N, C))
    p = _params(C)
    y, _ = block.forward(x, p, H, mode, l, c)
    dx, g = block.backward(x, dy, p, H, mode, l, c)
    ty, tdx, tg = _torch_block(x, dy, p, H, mode, l, c)
    np.testing.assert_allclose(y, ty, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(dx, tdx, rtol=1e-9, atol=1e-9)
    for k in p:
        np.testing.assert_allclose(g[k], tg[k], rtol=1e-9, atol=1e-9, err_msg=k)


def test_block_finite_differences():
    mode, B, N, H, D, l, c = "strided", 1, 16, 2, 4, 4, 0
    C = H * D
    rng = np.random.default_rng(1)
    x = rng.standard_normal((B, N, C))
    dy = rng.standard_normal((B, N, C))
    p = _params(C)
    dx, g = block.backward(x, dy, p, H, mode, l, c)

    def loss(xx, pp):
        return float((block.forward(xx, pp, H, mode, l, c)[0] * dy).sum())

    eps = 1e-6
    for idx in [(0, 0, 0), (0, 7, 3), (0, 15, 7)]:
        xp, xm = x.copy(), x.copy()
        xp[idx] += eps
        xm[idx] -= eps
        assert abs((loss(xp, p) - loss(xm, p)) / (2 * eps) - dx[idx]) < 1e-6 * max(1.0, abs(dx[idx]))
    for k, idx in [("w_qkv", (3, 17)), ("w_o", (5, 2)), ("w_1", (1, 30)), ("w_2", (29, 6)),
                   ("ln1_g", (4,)), ("ln1_b", (0,)), ("ln2_g", (7,)), ("ln2_b", (3,))]:
        pp, pm = dict(p), dict(p)
        pp[k] = p[k].copy()
        pm[k] = p[k].copy()
        pp[k][idx] += eps
        pm[k][idx] -= eps
        fd = (loss(x, pp) - loss(x, pm)) / (2 * eps)
        assert abs(fd - g[k][idx]) < 1e-6 * max(1.0, abs(fd)), k


def test_zero_output_projections_give_the_identity():
    mode, B, N, H, D, l, c = "fixed", 1, 32, 2, 8, 8, 2
    C = H * D
    rng = np.random.default_rng(2)
    x = rng.standard_normal((B, N, C))
    dy = rng.standard_normal((B, N, C))
    p = _params(C)
    p["w_o"] = np.zeros_like(p["w_o"])
    p["w_2"] = np.zeros_like(p["w_2"])
    y, _ = block.forward(x, p, H, mode, l, c)
    dx, g = block.backward(x, dy, p, H, mode, l, c)
    assert np.array_equal(y, x)
    assert np.array_equal(dx, dy)
    for k in ("w_qkv", "w_1", "ln1_g", "ln1_b", "ln2_g", "ln2_b"):
        assert not g[k].any(), k  # nothing reaches them through the zero projections


def test_layer_norm_and_gelu_closed_forms():
    g = np.linspace(0.5, 1.5, 8)
    b = np.linspace(-1.0, 1.0, 8)
    assert np.allclose(block.layer_norm(np.full((3, 8), 2.5), g, b), b)
    x = np.random.default_rng(3).standard_normal((5, 8))
    y = block.layer_norm(x, np.ones(8), np.zeros(8))
    assert np.allclose(y.mean(-1), 0) and np.allclose(y.var(-1), 1 / (1 + 1e-5 / x.var(-1)))
    assert block.gelu(np.array([0.0]))[0] == 0.0 and block.gelu_grad(np.array([0.0]))[0] == 0.5
    assert np.allclose(block.gelu(np.array([12.0])), 12.0) and np.allclose(block.gelu_grad(np.array([12.0])), 1.0)
    assert np.allclose(block.gelu(np.array([-12.0])), 0.0, atol=1e-30)

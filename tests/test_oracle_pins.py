"""Pins of the float64 oracle against things other than itself (CPU only).

* dense causal mode == torch's scaled_dot_product_attention in float64,
  gradients == torch autograd (a library routine, independent code);
* every mode: attention with the oracle's mask == library attention with
  the same mask, gradients == autograd;
* central finite differences of sum(O * dO) == analytic gradients;
* row sums of P, sum_j dV_j == sum_i dO_i, sum_j dK_j == 0.
"""

import numpy as np
import pytest
import torch

from oracle import attention, patterns
from factorized_block_sparse_b200 import synth

MODES = ("all", "local", "strided", "fixed")


def _block_mask(N, b, seed, p=0.4):
    """A caller block mask (lower blocks kept at random, diagonal always)."""
    rng = np.random.default_rng(seed)
    rp, ci = [0], []
    for r in range(N // b):
        ci += [s for s in range(r) if rng.random() < p] + [r]
        rp.append(len(ci))
    return patterns.BlockMask(N, b, rp, ci)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _torch_attention(q, k, v, dO, mask):
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    tm = torch.tensor(mask)
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=tm)
    out.backward(torch.tensor(dO))
    return out.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def test_all_mode_equals_library_causal_attention():
    B, H, N, D = 2, 3, 67, 16
    q, k, v, dO = (_rand((B, H, N, D), s) for s in range(4))
    O, lse = attention.forward(q, k, v, "all")
    dq, dk, dv = attention.backward(q, k, v, dO, "all", lse=lse)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    ref.backward(torch.tensor(dO))
    np.testing.assert_allclose(O, ref.detach().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-10, atol=1e-11)
    # lse against a library log-sum-exp over the causal row
    S = np.einsum("bhid,bhjd->bhij", q, k) / np.sqrt(D)
    S = np.where(np.tril(np.ones((N, N), bool)), S, -np.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(torch.tensor(S), -1).numpy(), rtol=1e-12)


@pytest.mark.parametrize("mode,l,c", [("local", 5, 0), ("strided", 6, 0), ("strided", 7, 0),
                                      ("fixed", 8, 2), ("fixed", 5, 1), ("column", 6, 0), ("block", 7, 0),
                                      (_block_mask(50, 5, 1), 1, 0)])
def test_sparse_modes_equal_library_masked_attention(mode, l, c):
    B, H, N, D = 1, 2, 50, 8
    q, k, v, dO = (_rand((B, H, N, D), 10 + s) for s in range(4))
    m = patterns.mask(mode, N, l, c)
    O, lse = attention.forward(q, k, v, mode, l, c)
    dq, dk, dv = attention.backward(q, k, v, dO, mode, l, c, lse=lse)
    rO, rq, rk, rv = _torch_attention(q, k, v, dO, m)
    for a, b in ((O, rO), (dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("mode,N,l,c", [("all", 16, 1, 0), ("local", 16, 4, 0),
                                        ("strided", 16, 4, 0), ("strided", 32, 4, 0),
                                        ("fixed", 16, 4, 1), ("fixed", 32, 4, 2), ("column", 16, 4, 0),
                                        ("block", 16, 4, 0), (_block_mask(16, 4, 2), 16, 1, 0)])
def test_finite_difference_gradients(mode, N, l, c):
    D = 8
    q, k, v, dO = (_rand((1, 1, N, D), 100 + s) for s in range(4))
    dq, dk, dv = attention.backward(q, k, v, dO, mode, l, c)

    def f(q_, k_, v_):
        O, _ = attention.forward(q_, k_, v_, mode, l, c)
        return float((O * dO).sum())

    h = 1e-6
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        num = np.zeros_like(grad)
        for idx in np.ndindex(grad.shape):
            args = {"q_": q.copy(), "k_": k.copy(), "v_": v.copy()}
            args[name + "_"][idx] += h
            fp = f(**args)
            args[name + "_"][idx] -= 2 * h
            fm = f(**args)
            num[idx] = (fp - fm) / (2 * h)
        rel = np.linalg.norm(num - grad) / np.linalg.norm(grad)
        assert rel <= 1e-6, (name, rel)


@pytest.mark.parametrize("mode,l,c", [("all", 1, 0), ("strided", 8, 0), ("fixed", 8, 3), ("column", 8, 0),
                                      ("block", 8, 0), (_block_mask(64, 8, 3), 1, 0)])
def test_invariants(mode, l, c):
    B, H, N, D = 1, 2, 64, 8
    q, k, v, dO = (_rand((B, H, N, D), 200 + s) for s in range(4))
    # rows of P sum to one: attention over v = 1 returns exactly 1
    O1, _ = attention.forward(q, k, np.ones_like(v), mode, l, c)
    np.testing.assert_allclose(O1, 1.0, rtol=0, atol=1e-13)
    dq, dk, dv = attention.backward(q, k, v, dO, mode, l, c)
    np.testing.assert_allclose(dv.sum(axis=2), dO.sum(axis=2), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)


@pytest.mark.parametrize("mode,l,c", [("strided", 16, 0), ("fixed", 16, 4), ("all", 1, 0), ("column", 16, 0),
                                      ("block", 16, 0), (_block_mask(96, 16, 4), 1, 0)])
def test_sampled_rows_and_columns_match_full(mode, l, c):
    B, H, N, D = 1, 2, 96, 8
    q, k, v, dO = (_rand((B, H, N, D), 300 + s) for s in range(4))
    O, lse = attention.forward(q, k, v, mode, l, c)
    dq, dk, dv = attention.backward(q, k, v, dO, mode, l, c, lse=lse)
    rows = np.array([0, 1, 15, 16, 17, 50, 95])
    Or, Lr = attention.forward_rows(q, k, v, mode, l, c, rows)
    np.testing.assert_allclose(Or, O[:, :, rows], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(Lr, lse[:, :, rows], rtol=1e-13)
    np.testing.assert_allclose(attention.dq_rows(q, k, v, dO, mode, l, c, rows),
                               dq[:, :, rows], rtol=1e-11, atol=1e-13)
    dkc, dvc = attention.dkv_cols(q, k, v, dO, mode, l, c, rows)
    np.testing.assert_allclose(dkc, dk[:, :, rows], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dvc, dv[:, :, rows], rtol=1e-11, atol=1e-13)


def test_synth_inputs_are_bf16_exact_and_seeded():
    x = synth.inputs(1, 2, 32, 8)
    y = synth.inputs(1, 2, 32, 8)
    for name in ("q", "k", "v", "dO"):
        assert str(x[name].dtype) == "torch.bfloat16"
        assert torch.equal(x[name], y[name])
        f = synth.to_f64(x[name])
        # widening bf16 -> f64 is exact: rounding the f64 back gives the same bits
        assert torch.equal(torch.tensor(f).to(torch.bfloat16), x[name])
    assert not torch.equal(x["q"], x["k"])

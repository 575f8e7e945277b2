"""Pins of the oracle's single-head modes ``column`` and ``block`` (CPU only).

The pages describe running the two parts of a factorized pattern as
separate heads, each with its own softmax ("OpenAI Sparse Transformer",
"Factorized Attention Patterns"; pcnews translation, "Разреженное
внимание").  The pins tie the two modes to the factorization, to closed
forms and to cases with a known answer:

* ``local`` | ``column`` is the strided mask and ``local``, ``column`` are
  its component heads; ``block`` is the fixed pattern's own-block head;
* nonzero counts equal closed forms;
* ``column`` with l >= N and ``block`` with l = 1 attend only to the
  position itself, so O = V and lse = s q.k exactly; ``column`` with l = 1
  and ``block`` with l >= N are dense causal;
* ``column`` in column-major order is attention with an inclusive
  block-diagonal triangle (row attention of the transposed array).
"""

import numpy as np
import pytest
import torch

from oracle import attention, patterns, views


@pytest.mark.parametrize("N,l", [(64, 8), (100, 7), (48, 48), (37, 5)])
def test_strided_is_local_or_column_and_those_are_its_heads(N, l):
    loc, col = patterns.mask("local", N, l), patterns.mask("column", N, l)
    assert np.array_equal(loc | col, patterns.mask("strided", N, l))
    A, B = patterns.component_heads("strided", N, l, 0)
    assert np.array_equal(A, loc) and np.array_equal(B, col)


@pytest.mark.parametrize("N,l,c", [(64, 8, 2), (96, 12, 5)])
def test_block_is_the_fixed_own_block_head(N, l, c):
    A, _ = patterns.component_heads("fixed", N, l, c)
    assert np.array_equal(patterns.mask("block", N, l), A)
    assert np.array_equal(patterns.mask("block", N, l) | patterns.mask("fixed", N, l, c),
                          patterns.mask("fixed", N, l, c))


@pytest.mark.parametrize("N,l", [(288, 12), (1024, 32), (96, 96)])
def test_nnz_closed_forms(N, l):
    m = N // l
    assert patterns.nnz("column", N, l) == N + l * m * (m - 1) // 2
    assert patterns.nnz("block", N, l) == m * l * (l + 1) // 2


def test_special_masks():
    N = 40
    tri = np.tril(np.ones((N, N), bool))
    eye = np.eye(N, dtype=bool)
    assert np.array_equal(patterns.mask("column", N, 1), tri)
    assert np.array_equal(patterns.mask("column", N, N), eye)
    assert np.array_equal(patterns.mask("column", N, N + 3), eye)
    assert np.array_equal(patterns.mask("block", N, N), tri)
    assert np.array_equal(patterns.mask("block", N, 1), eye)


@pytest.mark.parametrize("mode,l", [("column", 64), ("block", 1)])
def test_self_only_attention_returns_v(mode, l):
    rng = np.random.default_rng(3)
    B, H, N, D = 1, 2, 48, 16
    q, k, v = (rng.standard_normal((B, H, N, D)) for _ in range(3))
    o, lse = attention.forward(q, k, v, mode, l)
    np.testing.assert_array_equal(o, v)
    np.testing.assert_allclose(lse, np.einsum("bhnd,bhnd->bhn", q, k) / np.sqrt(D), rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("N,l", [(96, 8), (64, 16)])
def test_column_view_is_inclusive_row_attention_of_transposed_array(N, l):
    R = N // l
    runs = np.kron(np.eye(l, dtype=bool), np.tril(np.ones((R, R), bool)))
    assert np.array_equal(views.view_mask("T", "column", N, l), runs)
    rng = np.random.default_rng(11)
    q, k, v = (rng.standard_normal((N, 8)) for _ in range(3))
    o = views.column_order(N, l)
    sd = torch.nn.functional.scaled_dot_product_attention
    out_t = sd(torch.tensor(q[o])[None], torch.tensor(k[o])[None], torch.tensor(v[o])[None],
               attn_mask=torch.tensor(runs)[None])[0].numpy()
    out_nat = sd(torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None],
                 attn_mask=torch.tensor(patterns.mask("column", N, l))[None])[0].numpy()
    np.testing.assert_allclose(out_t[np.argsort(o)], out_nat, rtol=1e-12, atol=1e-13)

"""Pins of the oracle's caller block mask (``BlockMask``, CPU only).

The "Insights: 희소 어텐션 (Sparse Attention)" page gives the sparsity pattern
of ``SparseAttention(q, k, v, mask)`` as a mask over blocks.  The pins tie
the oracle's reading (element (i, j) kept when its block is and j <= i) to
independent constructions:

* all lower blocks is dense causal attention; diagonal blocks only is the
  block-diagonal causal mask (the ``block`` mode); a band of w blocks has a
  closed form;
* the element mask equals the Kronecker expansion of the block matrix
  intersected with the causal triangle, and attention through the oracle
  equals torch's SDPA with that mask;
* the natural-view block table of a mask is the caller's list, with the
  diagonal blocks PARTIAL and the others FULL;
* malformed lists (a missing diagonal, a block above it, unsorted columns)
  are refused.
"""

import numpy as np
import pytest
import torch

from oracle import attention, patterns, views


def _lower(nb, keep):
    rp, ci = [0], []
    for r in range(nb):
        ci += [s for s in range(r + 1) if keep(r, s)]
        rp.append(len(ci))
    return rp, ci


def test_all_lower_blocks_is_dense_causal():
    N, b = 96, 16
    bm = patterns.BlockMask(N, b, *_lower(N // b, lambda r, s: True))
    assert np.array_equal(patterns.mask(bm, N), patterns.mask("all", N))


def test_diagonal_only_is_the_block_head():
    N, b = 96, 16
    bm = patterns.BlockMask(N, b, *_lower(N // b, lambda r, s: r == s))
    assert np.array_equal(patterns.mask(bm, N), patterns.mask("block", N, b))


def test_band_closed_form():
    N, b, w = 128, 8, 3
    bm = patterns.BlockMask(N, b, *_lower(N // b, lambda r, s: r - s < w))
    i, j = np.arange(N)[:, None], np.arange(N)[None, :]
    assert np.array_equal(patterns.mask(bm, N), (j <= i) & (i // b - j // b < w))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_mask_is_kron_of_blocks_and_attention_matches_sdpa(seed):
    rng = np.random.default_rng(seed)
    N, b, D = 64, 8, 16
    nb = N // b
    keep = rng.random((nb, nb)) < 0.4
    bm = patterns.BlockMask(N, b, *_lower(nb, lambda r, s: r == s or keep[r, s]))
    blocks = np.tril(keep, -1) | np.eye(nb, dtype=bool)
    ref = np.kron(blocks, np.ones((b, b), bool)) & np.tril(np.ones((N, N), bool))
    assert np.array_equal(patterns.mask(bm, N), ref)
    q, k, v = (rng.standard_normal((1, 2, N, D)) for _ in range(3))
    o, _ = attention.forward(q, k, v, bm)
    sd = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k), torch.tensor(v), attn_mask=torch.tensor(ref)).numpy()
    np.testing.assert_allclose(o, sd, rtol=1e-12, atol=1e-13)


def test_block_table_is_the_callers_list():
    N, b = 96, 16
    rp, ci = _lower(N // b, lambda r, s: (r + s) % 3 != 1 or r == s)
    tab = views.block_table("N", patterns.BlockMask(N, b, rp, ci), N, 1, 0, b)
    assert tab["row_ptr"].tolist() == rp and tab["col_idx"].tolist() == ci
    rows = np.repeat(np.arange(N // b), np.diff(rp))
    assert tab["kind"].tolist() == [1 if c == r else 0 for r, c in zip(rows, ci)]


@pytest.mark.parametrize("rp,ci", [
    ([0, 1, 2], [0, 0]),        # row 1 lacks its diagonal block
    ([0, 1, 3], [0, 1, 0]),     # unsorted columns
    ([0, 2, 3], [0, 1, 1]),     # a block above the diagonal
])
def test_malformed_lists_are_refused(rp, ci):
    with pytest.raises(ValueError):
        patterns.BlockMask(32, 16, rp, ci)

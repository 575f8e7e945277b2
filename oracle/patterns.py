"""Element-level attention masks (float64 oracle; test infrastructure only).

A mask is a boolean matrix ``M[i, j]``: query position ``i`` may attend to
key position ``j``.  Every mode is causal and includes the diagonal, so no
query row is empty.

Definitions, and the reading of the pages they follow:

* ``all``     - ordinary dense causal attention, ``j <= i``.  This is the
  N x N attention the pages start from ("OpenAI Sparse Transformer",
  "Reducing Memory Constraints with Deep Attention"; the "all" mode of the
  ``attention_impl`` function on the "Insights: 희소 어텐션" page).
* ``local``   - a fixed window before ``i`` ("Insights" page, the window
  pattern and the "local" mode).  Reading: a window of ``l`` positions
  that includes ``i`` itself, ``0 <= i - j < l``.
* ``strided`` - each position attends to its own row and its own column
  when the sequence is laid out as a 2-D array with rows of length ``l``
  ("OpenAI Sparse Transformer", "Factorized Attention Patterns", strided
  bullet; pcnews translation, "Разреженное внимание").  Reading: the
  previous ``l`` positions (``0 <= i - j < l``) together with every earlier
  position in the same column, ``(i - j) mod l == 0``.  One head over the
  union, one softmax.
* ``fixed``   - fixed "summary" columns plus the elements of the current
  block (same sections, fixed bullet).  Reading: the own ``l``-block
  (``j // l == i // l``) together with the last ``c`` offsets of every
  block (``j mod l >= l - c``), causal.

The two component heads of each factorized pattern (used for the
two-step reachability property of "Factorized Attention Patterns") are
exposed as ``component_heads``.  The pages also describe running the two
parts as separate heads, each with its own softmax (same section: heads
that attend to the row and to the column, or to the own block and to the
summary cells).  Two of those heads are modes of their own:

* ``column``  - the strided pattern's column head: every earlier position
  of the same column and the position itself, ``(i - j) mod l == 0``.
  Its row head is ``local``.
* ``block``   - the fixed pattern's own-block head, ``j // l == i // l``,
  causal.
Both contain the diagonal, so no row is empty.

A caller's own block mask (the ``SparseAttention(q, k, v, mask)`` form of
the "Insights: 희소 어텐션" page, where the sparsity pattern is given as a
mask of blocks) is a ``BlockMask``: element (i, j) is in the mask when its
block (i // b, j // b) is and j <= i.  It stands wherever a mode string does.
"""

import numpy as np

MODES = ("all", "local", "strided", "fixed", "column", "block")


class BlockMask:
    """Lower-triangular block mask of an N-position sequence in blocks of ``b``.

    ``row_ptr`` / ``col_idx`` list, per query block r, the key blocks s <= r
    in the mask (ascending); every row holds its diagonal block, so no row
    is empty.  Element (i, j) is in the mask when block (i // b, j // b) is
    and j <= i.
    """

    def __init__(self, N, block, row_ptr, col_idx):
        if N % block:
            raise ValueError("N must be a multiple of block")
        nb = N // block
        row_ptr = np.asarray(row_ptr, dtype=np.int64)
        col_idx = np.asarray(col_idx, dtype=np.int64)
        if len(row_ptr) != nb + 1 or row_ptr[0] != 0 or row_ptr[-1] != len(col_idx):
            raise ValueError("row_ptr does not describe the column list")
        self.N, self.block = int(N), int(block)
        self.blocks = np.zeros((nb, nb), dtype=bool)
        for r in range(nb):
            cols = col_idx[row_ptr[r]:row_ptr[r + 1]]
            if len(cols) == 0 or cols[-1] != r or np.any(np.diff(cols) <= 0) or cols[0] < 0:
                raise ValueError(f"block row {r}: ascending columns <= {r} ending with the diagonal")
            self.blocks[r, cols] = True

    def pairs(self, i, j):
        i = np.asarray(i, dtype=np.int64)
        j = np.asarray(j, dtype=np.int64)
        return (j <= i) & self.blocks[i // self.block, j // self.block]


def _check(mode, N, l, c):
    if isinstance(mode, BlockMask):
        if N != mode.N:
            raise ValueError("block mask built for another N")
        return
    if mode not in MODES:
        raise ValueError(f"unknown mode {mode!r}")
    if N < 1:
        raise ValueError("N must be >= 1")
    if mode in ("local", "strided", "fixed", "column", "block") and l < 1:
        raise ValueError("l must be >= 1")
    if mode == "fixed" and not (0 <= c <= l):
        raise ValueError("fixed needs 0 <= c <= l")


def pair_mask(mode, l, c, i, j):
    """Membership of the pairs (i, j) (broadcasting integer arrays)."""
    if isinstance(mode, BlockMask):
        return mode.pairs(i, j)
    i = np.asarray(i, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    causal = j <= i
    if mode == "all":
        return causal
    d = i - j
    if mode == "local":
        return causal & (d < l)
    if mode == "strided":
        return causal & ((d < l) | (d % l == 0))
    if mode == "fixed":
        return causal & ((j // l == i // l) | (j % l >= l - c))
    if mode == "column":
        return causal & (d % l == 0)
    if mode == "block":
        return causal & (j // l == i // l)
    raise ValueError(f"unknown mode {mode!r}")


def mask_rows(mode, N, l, c, rows):
    """Boolean mask ``M[rows, :]`` of shape ``(len(rows), N)``."""
    _check(mode, N, l, c)
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(N, dtype=np.int64)[None, :]
    return pair_mask(mode, l, c, i, j)


def mask_cols(mode, N, l, c, cols):
    """Boolean mask ``M[:, cols]`` of shape ``(N, len(cols))``."""
    _check(mode, N, l, c)
    i = np.arange(N, dtype=np.int64)[:, None]
    j = np.asarray(cols, dtype=np.int64)[None, :]
    return pair_mask(mode, l, c, i, j)


def mask(mode, N, l=1, c=0):
    """The full ``N x N`` boolean mask (small N only)."""
    return mask_rows(mode, N, l, c, np.arange(N))


def component_heads(mode, N, l, c):
    """The two sparse heads whose composition the factorization relies on.

    strided: A = the previous ``l`` positions (row head), B = same column
    (column head).  fixed: A = own ``l``-block, B = summary columns.  Both
    are causal; the pattern's own mask is ``A | B``.
    """
    i = np.arange(N, dtype=np.int64)[:, None]
    j = np.arange(N, dtype=np.int64)[None, :]
    causal = j <= i
    if mode == "strided":
        A = causal & (i - j < l)
        B = causal & ((i - j) % l == 0)
    elif mode == "fixed":
        A = causal & (j // l == i // l)
        B = causal & (j % l >= l - c)
    else:
        raise ValueError("component heads exist for strided and fixed only")
    return A, B


def nnz(mode, N, l=1, c=0, chunk=4096):
    """Number of (i, j) pairs in the mask, counted row chunk by row chunk."""
    total = 0
    for r0 in range(0, N, chunk):
        rows = np.arange(r0, min(N, r0 + chunk))
        total += int(mask_rows(mode, N, l, c, rows).sum())
    return total

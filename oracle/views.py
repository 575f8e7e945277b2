"""Views of a factorized pattern and its block look-up tables (oracle).

Test infrastructure only (see the package docstring).

A block-sparse kernel slices queries and keys into blocks and works only
on the blocks that hold part of the mask ("OpenAI Sparse Transformer",
"Implementation and Limitations"; pcnews translation, "Релиз кода").  A
factorized pattern is not block-dense in one ordering, so it is split
into disjoint views, each dense in its own relabelled order:

* view ``N`` (natural order, queries and keys): ``all`` -> ``j <= i``;
  ``local`` and ``strided`` -> ``0 <= i - j < l``; ``fixed`` -> same
  ``l``-block, ``j <= i``.
* view ``T`` (strided only, the column part).  Attending along a column is
  attending along a row of the transposed 2-D array (pcnews translation,
  "Разреженное внимание", the parenthetical remark).  Queries and keys
  are relabelled into column-major order: position ``p`` sits at
  ``t(p) = (p mod l) * R + p // l`` with ``R = N / l`` (for ``N mod l != 0``
  the same column-major order, taken by sorting).  The view holds the
  strictly earlier positions of the same column, ``i - j > 0`` and
  ``(i - j) mod l == 0``; strictness keeps it disjoint from view ``N``,
  which already holds ``j == i``.
* view ``S`` (fixed only, the summary part).  Queries in natural order;
  keys restricted to the summary positions ``j mod l >= l - c`` and
  renumbered consecutively, ``sigma(j) = (j // l) * c + (j mod l - (l - c))``.
  The view holds the summary keys of strictly earlier blocks,
  ``j // l < i // l``.  Summary keys of the own block are in view ``N``.

The two single-head modes use one view each: ``column`` the column-major
view ``T`` with the diagonal included (``i - j >= 0``, ``(i - j) mod l ==
0``: there is no natural view to hold it), ``block`` the natural view of
``fixed``.  A caller's ``BlockMask`` is one natural view.

Block table of a view: cut its (queries x keys) matrix, in view order,
into ``block x block`` tiles (a ragged last tile is padded with
"not in mask").  A tile is present when any element is in the mask; it
is FULL (kind 0) when every element is, PARTIAL (kind 1) otherwise.
Each table is a CSR over query blocks with ascending key-block columns;
the transposed CSR (key-block major) serves the backward pass.
"""

import numpy as np

from .patterns import MODES, BlockMask

VIEWS = ("N", "T", "S")
FULL, PARTIAL = 0, 1


def views_of(mode):
    """Which views a mode is split into."""
    if isinstance(mode, BlockMask):
        return ("N",)
    if mode not in MODES:
        raise ValueError(mode)
    if mode == "strided":
        return ("N", "T")
    if mode == "fixed":
        return ("N", "S")
    if mode == "column":
        return ("T",)
    return ("N",)


def column_order(N, l):
    """Natural positions listed in column-major (transposed) order."""
    p = np.arange(N, dtype=np.int64)
    return np.lexsort((p // l, p % l))


def summary_order(N, l, c):
    """Natural positions of the summary keys, in their consecutive order."""
    p = np.arange(N, dtype=np.int64)
    return p[(p % l) >= (l - c)]


def _natural_view_predicate(view, mode, l, c, i, j):
    """Membership of natural pair (i, j) in a view (broadcasting arrays)."""
    causal = j <= i
    if view == "N":
        if isinstance(mode, BlockMask):
            return mode.pairs(i, j)
        if mode == "all":
            return causal
        if mode in ("local", "strided"):
            return causal & (i - j < l)
        return causal & (j // l == i // l)  # fixed, block
    if view == "T":
        d = i - j
        if mode == "column":
            return (d >= 0) & (d % l == 0)
        return (d > 0) & (d % l == 0)
    if view == "S":
        return (j // l < i // l) & (j % l >= l - c)
    raise ValueError(view)


def view_shape(view, mode, N, l, c):
    """(number of query positions, number of key positions) of a view."""
    if view == "S":
        return N, len(summary_order(N, l, c))
    return N, N


def view_mask_rows(view, mode, N, l, c, rows):
    """Rows ``rows`` (view order) of the view's mask, keys in view order."""
    rows = np.asarray(rows, dtype=np.int64)
    if view == "T":
        order = column_order(N, l)
        qi = order[rows]
        kj = order
    elif view == "S":
        qi = rows
        kj = summary_order(N, l, c)
    else:
        qi = rows
        kj = np.arange(N, dtype=np.int64)
    return _natural_view_predicate(view, mode, l, c, qi[:, None], kj[None, :])


def view_mask(view, mode, N, l=1, c=0):
    return view_mask_rows(view, mode, N, l, c, np.arange(view_shape(view, mode, N, l, c)[0]))


def block_table(view, mode, N, l, c, block, rows=None, chunk_rows=4096):
    """CSR block table of one view by block-OR (any) / block-AND (all).

    Returns ``dict(row_ptr, col_idx, kind, n_rows, n_cols)``.  With
    ``rows`` (a list of query-block indices) only those block rows are
    evaluated, and ``row_ptr`` indexes the returned subset.
    """
    nq, nk = view_shape(view, mode, N, l, c)
    if nq % block:
        raise ValueError("N must be a multiple of block")
    n_rows = nq // block
    n_cols = -(-nk // block)
    pad = n_cols * block - nk
    sel = np.arange(n_rows) if rows is None else np.asarray(rows, dtype=np.int64)
    per_chunk = max(1, chunk_rows // block)
    row_ptr = [0]
    cols, kinds = [], []
    for s0 in range(0, len(sel), per_chunk):
        brs = sel[s0:s0 + per_chunk]
        q = (brs[:, None] * block + np.arange(block)[None, :]).reshape(-1)
        m = view_mask_rows(view, mode, N, l, c, q)
        if pad:
            m = np.concatenate([m, np.zeros((len(q), pad), dtype=bool)], axis=1)
        m = m.reshape(len(brs), block, n_cols, block)
        anyb = m.any(axis=(1, 3))
        allb = m.all(axis=(1, 3))
        for r in range(len(brs)):
            cc = np.nonzero(anyb[r])[0]
            cols.append(cc.astype(np.int32))
            kinds.append(np.where(allb[r, cc], FULL, PARTIAL).astype(np.uint8))
            row_ptr.append(row_ptr[-1] + len(cc))
    return dict(
        row_ptr=np.asarray(row_ptr, dtype=np.int32),
        col_idx=np.concatenate(cols) if cols else np.zeros(0, np.int32),
        kind=np.concatenate(kinds) if kinds else np.zeros(0, np.uint8),
        n_rows=n_rows if rows is None else len(sel),
        n_cols=n_cols,
    )


def transpose_table(tab):
    """Key-block-major CSR of a block table (ascending query blocks)."""
    n_rows, n_cols = tab["n_rows"], tab["n_cols"]
    rp, ci, kd = tab["row_ptr"], tab["col_idx"], tab["kind"]
    per = [[] for _ in range(n_cols)]
    for r in range(n_rows):
        for e in range(rp[r], rp[r + 1]):
            per[ci[e]].append((r, kd[e]))
    row_ptr = [0]
    cols, kinds = [], []
    for cidx in range(n_cols):
        for r, k in per[cidx]:
            cols.append(r)
            kinds.append(k)
        row_ptr.append(len(cols))
    return dict(
        row_ptr=np.asarray(row_ptr, dtype=np.int32),
        col_idx=np.asarray(cols, dtype=np.int32),
        kind=np.asarray(kinds, dtype=np.uint8),
        n_rows=n_cols,
        n_cols=n_rows,
    )


def block_nonzeros(mode, N, l, c, block):
    """Number of present blocks per view (the public table's nnz)."""
    return {v: int(len(block_table(v, mode, N, l, c, block)["col_idx"])) for v in views_of(mode)}

"""Masked softmax attention and its analytic gradient in float64 (oracle).

Test infrastructure only (see the package docstring).

What is computed (per batch b and head h, shapes ``[B, H, N, D]``):

* scores ``S_ij = s * <q_i, k_j>`` on the mask, ``-inf`` elsewhere, with
  ``s = 1/sqrt(D)`` (the pages say only "dot product, then softmax" -
  "Insights: 희소 어텐션" page; the 1/sqrt(D) scale is the reading taken);
* ``lse_i = log sum_j exp S_ij`` (natural log), ``P = exp(S - lse)``,
  ``O = P V``;
* backward for an upstream gradient ``dO``: ``dV = P^T dO``,
  ``dP = dO V^T``, ``D_i = sum_j P_ij dP_ij``, ``dS = P * (dP - D)``,
  ``dQ = s dS K``, ``dK = s dS^T Q``.  The backward recomputes ``P`` from
  ``lse`` instead of keeping it, the memory-saving recomputation of the
  pages ("Generating Long Sequences with Sparse Transformers", ABSTRACT,
  item b; pcnews translation, "Глубокое внимание").

The mask of each row chunk is formed explicitly from the element
predicate (``oracle.patterns``), so the whole ``N x N`` mask is never held.
Sampled variants compute selected query rows (``O``, ``lse``, ``dQ``) or
selected key columns (``dK``, ``dV``) from the same definitions, for
comparisons at sizes where the whole oracle would take too long.
"""

import numpy as np

from . import patterns


def _scale(D, scale):
    return 1.0 / np.sqrt(D) if scale is None else float(scale)


def _chunk(N, chunk):
    if chunk is not None:
        return chunk
    return max(1, min(512, (1 << 23) // max(N, 1)))


def _rows_softmax(qh, kh, mode, l, c, rows, s):
    """Masked scores of ``rows`` -> (P, lse) for one (b, h)."""
    N = kh.shape[0]
    m = patterns.mask_rows(mode, N, l, c, rows)
    S = (qh[rows] @ kh.T) * s
    S = np.where(m, S, -np.inf)
    mx = S.max(axis=1, keepdims=True)
    E = np.exp(S - mx)
    tot = E.sum(axis=1, keepdims=True)
    lse = (mx + np.log(tot))[:, 0]
    P = E / tot
    return P, lse


def forward(q, k, v, mode, l=1, c=0, scale=None, chunk=None):
    """Full forward: returns ``(O, lse)`` with shapes ``[B,H,N,D]``, ``[B,H,N]``."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, H, N, D = q.shape
    s = _scale(D, scale)
    O = np.zeros_like(q)
    L = np.zeros((B, H, N))
    ch = _chunk(N, chunk)
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, ch):
                rows = np.arange(r0, min(N, r0 + ch))
                P, lse = _rows_softmax(q[b, h], k[b, h], mode, l, c, rows, s)
                O[b, h, rows] = P @ v[b, h]
                L[b, h, rows] = lse
    return O, L


def backward(q, k, v, dO, mode, l=1, c=0, scale=None, lse=None, chunk=None):
    """Full backward: returns ``(dQ, dK, dV)``.

    ``lse`` is recomputed when not given.  ``D_i`` is formed from ``P``
    and ``dP`` by its definition.
    """
    q, k, v, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dO))
    B, H, N, D = q.shape
    s = _scale(D, scale)
    if lse is None:
        _, lse = forward(q, k, v, mode, l, c, scale, chunk)
    dQ = np.zeros_like(q)
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    ch = _chunk(N, chunk)
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, ch):
                rows = np.arange(r0, min(N, r0 + ch))
                m = patterns.mask_rows(mode, N, l, c, rows)
                S = np.where(m, (q[b, h, rows] @ k[b, h].T) * s, -np.inf)
                P = np.exp(S - lse[b, h, rows][:, None])
                dV[b, h] += P.T @ dO[b, h, rows]
                dP = dO[b, h, rows] @ v[b, h].T
                Di = (P * dP).sum(axis=1, keepdims=True)
                dS = P * (dP - Di)
                dQ[b, h, rows] = s * (dS @ k[b, h])
                dK[b, h] += s * (dS.T @ q[b, h, rows])
    return dQ, dK, dV


def forward_rows(q, k, v, mode, l, c, rows, scale=None):
    """``O[:, :, rows]`` and ``lse[:, :, rows]`` only."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, H, N, D = q.shape
    s = _scale(D, scale)
    rows = np.asarray(rows, dtype=np.int64)
    O = np.zeros((B, H, len(rows), D))
    L = np.zeros((B, H, len(rows)))
    for b in range(B):
        for h in range(H):
            P, lse = _rows_softmax(q[b, h], k[b, h], mode, l, c, rows, s)
            O[b, h] = P @ v[b, h]
            L[b, h] = lse
    return O, L


def _row_grads(qh, kh, vh, dOh, mode, l, c, rows, s):
    """P, dS of the given rows of one (b, h)."""
    P, _ = _rows_softmax(qh, kh, mode, l, c, rows, s)
    dP = dOh[rows] @ vh.T
    Di = (P * dP).sum(axis=1, keepdims=True)
    return P, P * (dP - Di)


def dq_rows(q, k, v, dO, mode, l, c, rows, scale=None):
    """``dQ[:, :, rows]`` only (each query row needs nothing but itself)."""
    q, k, v, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dO))
    B, H, N, D = q.shape
    s = _scale(D, scale)
    rows = np.asarray(rows, dtype=np.int64)
    out = np.zeros((B, H, len(rows), D))
    for b in range(B):
        for h in range(H):
            _, dS = _row_grads(q[b, h], k[b, h], v[b, h], dO[b, h], mode, l, c, rows, s)
            out[b, h] = s * (dS @ k[b, h])
    return out


def dkv_cols(q, k, v, dO, mode, l, c, cols, scale=None, chunk=None):
    """``dK[:, :, cols]`` and ``dV[:, :, cols]`` only.

    Only the query rows whose mask row contains one of ``cols`` contribute;
    each of them is evaluated in full (its softmax needs the whole row).
    """
    q, k, v, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dO))
    B, H, N, D = q.shape
    s = _scale(D, scale)
    cols = np.asarray(cols, dtype=np.int64)
    seen = patterns.mask_cols(mode, N, l, c, cols).any(axis=1)
    rows_all = np.nonzero(seen)[0]
    dK = np.zeros((B, H, len(cols), D))
    dV = np.zeros((B, H, len(cols), D))
    ch = _chunk(N, chunk)
    for b in range(B):
        for h in range(H):
            for r0 in range(0, len(rows_all), ch):
                rows = rows_all[r0:r0 + ch]
                P, dS = _row_grads(q[b, h], k[b, h], v[b, h], dO[b, h], mode, l, c, rows, s)
                dV[b, h] += P[:, cols].T @ dO[b, h, rows]
                dK[b, h] += s * (dS[:, cols].T @ q[b, h, rows])
    return dK, dV

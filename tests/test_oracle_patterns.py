"""Pins of the oracle's masks, views and block tables (CPU only).

* two-step reachability through the two factorized heads ("OpenAI Sparse
  Transformer", "Factorized Attention Patterns": every position is reached
  in two sparse-attention steps);
* nonzero counts equal closed forms derived from the pattern definitions
  and grow as O(N sqrt N) with l = floor(sqrt N) ("Sparse Attention and
  Algorithmic Complexity");
* special cases that reduce to dense causal or block-diagonal attention;
* the column view is row attention on the transposed array (pcnews
  translation, "Разреженное внимание"): attention computed in relabelled
  order equals attention with the natural-order column mask;
* block tables equal a brute-force per-element walk on tiny inputs, and
  the per-config table sizes in ``tests/golden/lut_counts.json``.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import patterns, views

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _reach_two_steps(A, B):
    Ai, Bi = A.astype(np.int64), B.astype(np.int64)
    return A | B | ((Ai @ Bi) > 0) | ((Bi @ Ai) > 0)


@pytest.mark.parametrize("N,l", [(64, 8), (100, 7), (256, 16), (250, 15), (37, 40)])
def test_strided_two_step_reachability(N, l):
    A, B = patterns.component_heads("strided", N, l, 0)
    assert np.array_equal(A | B, patterns.mask("strided", N, l, 0))
    assert np.array_equal(_reach_two_steps(A, B), np.tril(np.ones((N, N), bool)))


@pytest.mark.parametrize("N,l,c", [(64, 8, 1), (100, 10, 3), (256, 16, 2), (250, 16, 4)])
def test_fixed_two_step_reachability(N, l, c):
    A, B = patterns.component_heads("fixed", N, l, c)
    assert np.array_equal(A | B, patterns.mask("fixed", N, l, c))
    assert np.array_equal(_reach_two_steps(A, B), np.tril(np.ones((N, N), bool)))


def test_fixed_without_summary_columns_does_not_reach_everything():
    A, B = patterns.component_heads("fixed", 64, 8, 0)
    assert not np.array_equal(_reach_two_steps(A, B), np.tril(np.ones((64, 64), bool)))


def _closed_form(mode, N, l, c):
    """Counts from the definitions, N a multiple of l (m = N / l rows)."""
    m = N // l
    if mode == "all":
        return N * (N + 1) // 2
    if mode == "local":
        return l * (l + 1) // 2 + (N - l) * l
    if mode == "strided":
        return l * (l + 1) // 2 + (N - l) * l + l * m * (m - 1) // 2
    if mode == "column":
        return N + l * m * (m - 1) // 2
    if mode == "block":
        return m * l * (l + 1) // 2
    return m * l * (l + 1) // 2 + c * l * m * (m - 1) // 2


@pytest.mark.parametrize("mode,N,l,c", [("all", 300, 1, 0), ("local", 300, 12, 0),
                                        ("strided", 288, 12, 0), ("strided", 1024, 32, 0),
                                        ("fixed", 288, 12, 3), ("fixed", 1024, 32, 8)])
def test_nnz_closed_forms(mode, N, l, c):
    assert patterns.nnz(mode, N, l, c) == _closed_form(mode, N, l, c)


def test_nnz_of_named_workloads():
    with open(os.path.join(GOLDEN, "nnz_counts.json")) as f:
        gold = json.load(f)
    for name, rec in gold["workloads"].items():
        assert _closed_form(rec["mode"], rec["N"], rec["l"], rec["c"]) == rec["nnz_per_head"], name
        if rec["N"] <= 12288:
            assert patterns.nnz(rec["mode"], rec["N"], rec["l"], rec["c"]) == rec["nnz_per_head"], name


def test_nnz_grows_as_n_sqrt_n():
    ratios = {"strided": [], "fixed": [], "all": []}
    for N in (256, 1024, 4096, 16384):
        l = int(np.sqrt(N))
        for mode in ratios:
            ratios[mode].append(patterns.nnz(mode, N, l, 8 if mode == "fixed" else 0) / N ** 1.5)
    for mode in ("strided", "fixed"):
        r = np.array(ratios[mode])
        assert r.max() / r.min() < 1.1, (mode, r)
    a = np.array(ratios["all"])
    assert np.all(a[1:] / a[:-1] > 1.9)  # dense causal: doubles per 4x N


def test_special_cases():
    N = 48
    tri = np.tril(np.ones((N, N), bool))
    for l in (N, N + 5):
        assert np.array_equal(patterns.mask("local", N, l, 0), tri)
        assert np.array_equal(patterns.mask("strided", N, l, 0), tri)
    assert np.array_equal(patterns.mask("strided", N, 1, 0), tri)
    assert np.array_equal(patterns.mask("fixed", N, 8, 8), tri)
    blockdiag = np.kron(np.eye(N // 8, dtype=bool), np.tril(np.ones((8, 8), bool)))
    assert np.array_equal(patterns.mask("fixed", N, 8, 0), blockdiag)
    # local is a band of width l including the diagonal
    band = tri & ~np.tril(np.ones((N, N), bool), -5)
    assert np.array_equal(patterns.mask("local", N, 5, 0), band)


def _sdpa(q, k, v, m):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k), torch.tensor(v), attn_mask=torch.tensor(m)).numpy()


@pytest.mark.parametrize("N,l", [(96, 8), (64, 16), (60, 6)])
def test_column_view_is_row_attention_of_transposed_array(N, l):
    rng = np.random.default_rng(7)
    q, k, v = (rng.standard_normal((N, 8)) for _ in range(3))
    order = views.column_order(N, l)
    # the relabelling puts each column of the 2-D array (rows of length l) in one run
    R = N // l
    assert np.array_equal(order.reshape(l, R), np.arange(N).reshape(R, l).T)
    # natural order: strictly earlier positions of the same column
    i, j = np.arange(N)[:, None], np.arange(N)[None, :]
    col = (i - j > 0) & ((i - j) % l == 0)
    # transposed order: strict causal inside each run of R (block-diagonal strict triangle)
    runs = np.kron(np.eye(l, dtype=bool), np.tril(np.ones((R, R), bool), -1))
    assert np.array_equal(views.view_mask("T", "strided", N, l), runs)
    live = col.any(axis=1)  # the first element of each column has no column keys
    out_nat = _sdpa(q[live][None], k[None], v[None], col[live][None])[0]
    tl = runs.any(axis=1)
    out_t = _sdpa(q[order][tl][None], k[order][None], v[order][None], runs[tl][None])[0]
    nat_rows = np.nonzero(live)[0]
    t_rows = order[np.nonzero(tl)[0]]
    srt = np.argsort(t_rows)
    assert np.array_equal(t_rows[srt], nat_rows)
    np.testing.assert_allclose(out_t[srt], out_nat, rtol=1e-12, atol=1e-13)


def test_summary_view_is_block_prefix():
    N, l, c = 96, 12, 3
    S = views.view_mask("S", "fixed", N, l, c)
    i = np.arange(N)[:, None]
    s = np.arange(S.shape[1])[None, :]
    assert S.shape == (N, (N // l) * c)
    assert np.array_equal(S, s < (i // l) * c)
    j = views.summary_order(N, l, c)
    assert np.array_equal(j, np.array([g * l + (l - c) + u for g in range(N // l) for u in range(c)]))


@pytest.mark.parametrize("mode,N,l,c", [("all", 64, 1, 0), ("local", 64, 6, 0),
                                        ("strided", 64, 8, 0), ("strided", 60, 6, 0),
                                        ("fixed", 64, 8, 2), ("fixed", 72, 12, 5),
                                        ("column", 64, 8, 0), ("column", 60, 6, 0), ("block", 64, 8, 0)])
def test_views_partition_the_mask(mode, N, l, c):
    full = patterns.mask(mode, N, l, c)
    acc = np.zeros((N, N), np.int64)
    for v in views.views_of(mode):
        M = views.view_mask(v, mode, N, l, c)
        if v == "T":
            o = views.column_order(N, l)
            nat = np.zeros((N, N), bool)
            nat[np.ix_(o, o)] = M
        elif v == "S":
            nat = np.zeros((N, N), bool)
            nat[:, views.summary_order(N, l, c)] = M
        else:
            nat = M
        acc += nat
    assert acc.max() <= 1  # disjoint
    assert np.array_equal(acc.astype(bool), full)


def _brute_table(M, b):
    nq, nk = M.shape
    rp, ci, kd = [0], [], []
    for r in range(nq // b):
        for cb in range(-(-nk // b)):
            vals = [bool(M[r * b + x, cb * b + y]) if cb * b + y < nk else False
                    for x in range(b) for y in range(b)]
            if any(vals):
                ci.append(cb)
                kd.append(0 if all(vals) else 1)
        rp.append(len(ci))
    return rp, ci, kd


@pytest.mark.parametrize("mode,N,l,c,b", [("all", 64, 1, 0, 8), ("local", 64, 12, 0, 8),
                                          ("strided", 64, 8, 0, 4), ("strided", 96, 12, 0, 8),
                                          ("fixed", 96, 12, 4, 8), ("fixed", 64, 16, 3, 4),
                                          ("column", 64, 8, 0, 4), ("column", 96, 12, 0, 8),
                                          ("block", 96, 12, 0, 8)])
def test_block_tables_brute_force(mode, N, l, c, b):
    for v in views.views_of(mode):
        tab = views.block_table(v, mode, N, l, c, b)
        rp, ci, kd = _brute_table(views.view_mask(v, mode, N, l, c), b)
        assert tab["row_ptr"].tolist() == rp
        assert tab["col_idx"].tolist() == ci
        assert tab["kind"].tolist() == kd
        tt = views.transpose_table(tab)
        rpt, cit, kdt = _brute_table(views.view_mask(v, mode, N, l, c).T.copy(), b)
        assert tt["row_ptr"].tolist() == rpt and tt["col_idx"].tolist() == cit
        assert tt["kind"].tolist() == kdt


def test_block_table_sizes_of_named_workloads():
    with open(os.path.join(GOLDEN, "lut_counts.json")) as f:
        gold = json.load(f)
    for name, rec in gold["workloads"].items():
        if rec["N"] > 12288:
            continue
        for v, (nfull, npart) in rec["views"].items():
            tab = views.block_table(v, rec["mode"], rec["N"], rec["l"], rec["c"], rec["block"])
            assert int((tab["kind"] == 0).sum()) == nfull, (name, v)
            assert int((tab["kind"] == 1).sum()) == npart, (name, v)


def test_pages_memory_figure():
    """A 64x64x3 image is N = 12288; 64 layers x 4 heads of N x N fp32 scores is ~154 GB
    ("OpenAI Sparse Transformer", "Reducing Memory Constraints with Deep Attention")."""
    with open(os.path.join(GOLDEN, "pages_numbers.json")) as f:
        gold = json.load(f)
    rec = gold["attention_matrix_memory"]
    N = rec["height"] * rec["width"] * rec["channels"]
    assert N == 12288
    nbytes = N * N * rec["layers"] * rec["heads"] * rec["bytes_per_element"]
    assert int(nbytes // 10**9) == rec["gigabytes"]  # 154.6e9 B, printed as 154 GB

"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Element by element at sizes the oracle finishes in seconds (several tiles
and ragged tails); at the named workloads' full sizes on sampled rows and
key columns that the oracle computes one by one.  Tolerances: max-abs 2e-2
and relative L2 5e-3 for O, dQ, dK, dV (bf16) and lse (fp32).
"""

import numpy as np
import pytest
import torch

from factorized_block_sparse_b200 import synth
from oracle import attention
from gpu_util import assert_close, oracle_full, run_library

pytestmark = pytest.mark.gpu

SMALL = [
    # mode, B, H, N, D, l, c, block
    ("strided", 1, 1, 256, 32, 16, 0, 16),      # the tiny workload, whole
    ("strided", 1, 2, 1024, 128, 32, 0, 32),    # image32-like: D=128, R=32 (4 columns per tile)
    ("strided", 2, 1, 2048, 64, 64, 0, 64),     # R=32
    ("strided", 1, 2, 2048, 64, 16, 0, 64),     # R=128: one column per tile
    ("strided", 1, 1, 4096, 64, 16, 0, 64),     # R=256: two tiles per column
    ("fixed", 1, 2, 2048, 64, 128, 32, 64),     # text-like
    ("fixed", 2, 1, 1536, 64, 96, 16, 32),      # l not a multiple of the tile
    ("fixed", 1, 1, 1024, 64, 128, 64, 64),     # c = 64
    ("fixed", 1, 1, 1024, 32, 128, 128, 64),    # c = l (dense causal)
    ("all", 1, 2, 1024, 64, 1, 0, 64),
    ("all", 1, 1, 320, 64, 1, 0, 64),           # ragged last tile (N % 128 != 0)
    ("local", 2, 1, 1024, 64, 100, 0, 16),      # window not aligned to blocks
    ("local", 1, 1, 512, 128, 1000, 0, 64),     # window wider than the sequence
    ("strided", 1, 1, 320, 64, 40, 0, 32),      # R = 8, ragged
    # items of >= 16 steps on average: the LONG backward shape (P^T in TMEM)
    ("all", 1, 1, 2112, 32, 1, 0, 64),          # D = 32, ragged last key tile
    ("all", 2, 1, 2112, 64, 1, 0, 64),
    # single-head modes: the strided column head and the fixed own-block head
    ("column", 1, 2, 2048, 64, 64, 0, 64),      # R = 32: four columns per 128-key tile
    ("column", 1, 1, 1024, 32, 8, 0, 32),       # R = 128: one column per tile
    ("column", 2, 1, 2048, 128, 16, 0, 64),     # D = 128, R = 128
    ("column", 1, 1, 4096, 64, 16, 0, 64),      # R = 256: two tiles per column
    ("block", 1, 2, 1024, 64, 128, 0, 64),
    ("block", 2, 1, 960, 32, 100, 0, 64),       # l does not divide N
    ("block", 1, 1, 1024, 128, 256, 0, 64),
    # strided with l = 192 (R = 16): the natural view's key tiles see about five
    # 64-query steps each, so its backward takes the LONG shape element by element
    ("strided", 1, 1, 3072, 64, 192, 0, 64),
    ("strided", 1, 2, 6144, 64, 192, 0, 64),    # R = 32, image64's row length
    # column and summary geometries that need TMA boxes of gcd(R, rows) or
    # gcd(c, rows) rows: R neither dividing nor divisible by 128, R odd, c
    # neither dividing 64 nor a multiple of 128
    ("strided", 1, 1, 1536, 64, 64, 0, 64),     # R = 24
    ("strided", 1, 2, 1280, 64, 256, 0, 64),    # R = 5
    ("column", 1, 1, 768, 64, 64, 0, 64),       # R = 12
    ("column", 1, 1, 1344, 64, 64, 0, 64),      # R = 21
    ("fixed", 1, 1, 2048, 64, 128, 48, 64),     # c = 48
    ("fixed", 1, 1, 1536, 32, 96, 24, 32),      # c = 24, D = 32
    ("fixed", 1, 2, 1024, 128, 128, 96, 64),    # c = 96, D = 128
    # N not a multiple of l (a partial last block)
    ("fixed", 1, 2, 1136, 64, 128, 32, 16),     # the partial block holds summary offsets of its own
    ("fixed", 2, 1, 1088, 32, 128, 16, 64),     # ... and here it does not
    ("fixed", 1, 1, 3000, 64, 128, 32, 8),      # summary view long enough for the LONG shape
    ("strided", 1, 2, 1000, 64, 64, 0, 8),      # R = 15 whole rows + a partial row of 40
    ("strided", 2, 1, 1216, 32, 96, 0, 64),     # R = 12 + 64, D = 32
    ("strided", 1, 1, 1152 + 80, 128, 96, 0, 16),  # R = 12 + 80, D = 128
    ("strided", 1, 1, 200, 64, 256, 0, 8),      # N < l: no whole row, no column part
    ("fixed", 1, 1, 200, 64, 256, 64, 8),       # N < l: one partial block, no summary view
    ("strided", 1, 1, 3000, 64, 192, 0, 8),     # R = 15 + 120, the natural view in the LONG shape
    # one key tile per query step in the natural view with no earlier pass:
    # the natural pass writes the final dQ alone (D = 128, ragged)
    ("block", 1, 1, 1088, 128, 128, 0, 64),
    ("block", 2, 1, 1000, 32, 64, 0, 8),
    # fixed with l = 512: natural items of 5 steps on average take the LONG shape, whose epilogue
    # loads the summary partials and adds them itself (the SHORT shape reduces into them instead)
    ("fixed", 1, 1, 2048, 64, 512, 64, 64),
    # summary rows of up to 127 steps (LONG items of many steps), and a ragged last block at D = 32
    ("fixed", 1, 1, 8192, 64, 64, 16, 64),
    ("fixed", 2, 1, 8100, 32, 64, 16, 4),       # ragged last block, D = 32
]


@pytest.mark.parametrize("mode,B,H,N,D,l,c,block", SMALL)
def test_parity_elementwise(cuda_device, mode, B, H, N, D, l, c, block):
    x, got, _ = run_library(mode, B, H, N, D, l, c, block)
    ref = oracle_full(x, mode, l, c)
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert np.isfinite(got[name]).all(), name
        assert_close(f"{mode} N={N} D={D} {name}", got[name], ref[name])


@pytest.mark.parametrize("mode,B,H,N,D,l,c,block,scale", [
    ("strided", 1, 2, 1024, 64, 32, 0, 64, 0.05),   # flat softmax
    ("fixed", 1, 1, 1024, 32, 128, 32, 64, 0.3),    # sharper than 1/sqrt(32)
    # the column head, whose rows have few keys: below the default 0.125, and
    # above it, where dK grows past |4| and bf16 rounding of the exact result
    # alone is up to 2^-6 (the bound is taken on top of the output's rounding)
    ("column", 1, 1, 1024, 64, 32, 0, 64, 0.1),
    ("column", 1, 1, 1024, 64, 32, 0, 64, 0.2),
])
def test_parity_explicit_scale(cuda_device, mode, B, H, N, D, l, c, block, scale):
    x, got, _ = run_library(mode, B, H, N, D, l, c, block, scale=scale)
    ref = oracle_full(x, mode, l, c, scale=scale)
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert np.isfinite(got[name]).all(), name
        assert_close(f"{mode} scale={scale} {name}", got[name], ref[name])


def test_default_scale_is_inverse_sqrt_d(cuda_device):
    # the plain entry points are the _ex ones with scale 1/sqrt(D), bit for bit
    a = run_library("fixed", 1, 1, 1024, 32, 128, 32, 64)[1]
    b = run_library("fixed", 1, 1, 1024, 32, 128, 32, 64, scale=1.0 / np.sqrt(32))[1]
    for name in ("o", "lse", "dk", "dv"):
        assert np.array_equal(a[name], b[name]), name


@pytest.mark.parametrize("mode,B,H,N,D,l,c,block", [
    ("strided", 1, 2, 2048, 64, 64, 0, 64),
    # fixed at N = 4096: its summary view's key tiles see about 30 query steps
    # each (the LONG backward shape, the text workload's dominant pass)
    ("fixed", 1, 2, 4096, 64, 128, 32, 64),
])
def test_dk_dv_deterministic(cuda_device, mode, B, H, N, D, l, c, block):
    a = run_library(mode, B, H, N, D, l, c, block)[1]
    b = run_library(mode, B, H, N, D, l, c, block)[1]
    for name in ("o", "lse", "dk", "dv"):
        assert np.array_equal(a[name], b[name]), name


def _tiles(N, n_mid, rng, extra=()):
    """Whole 128-position tiles: the first, the last, n_mid random ones and the
    tiles holding the positions in ``extra``; returns sorted positions."""
    n_t = (N + 127) // 128
    ts = {0, n_t - 1, *rng.integers(0, n_t, n_mid).tolist(), *(int(p) // 128 for p in extra)}
    return np.concatenate([np.arange(t * 128, min(N, t * 128 + 128)) for t in sorted(ts)])


def _sampled(name, n_mid=2, slices=((0, 0),), seed=0):
    """Whole 128-row query tiles (O, lse, dQ) and whole 128-key key tiles (dK,
    dV) of a full-size workload against the oracle, which computes them one
    row or key column at a time: the first and last tiles, random ones and,
    for the fixed pattern, key tiles holding summary keys of an early and a
    late block."""
    w = synth.WORKLOADS[name]
    mode, B, H, N, D, l, c, block = (w[k] for k in ("mode", "B", "H", "N", "D", "l", "c", "block"))
    x, got, _ = run_library(mode, B, H, N, D, l, c, block)
    rng = np.random.default_rng(seed)
    rows = _tiles(N, n_mid, rng)
    extra = [l - 1, (N // l - 2) * l + l - c] if mode == "fixed" else []
    if N <= 16384:
        cols = _tiles(N, n_mid, rng, extra)
    else:  # an early key is seen by ~N/l column rows of N keys each: the last tile + single columns
        cols = np.unique(np.concatenate([[0, 1], rng.integers(0, N, 8), np.arange(N - 128, N)]))
    for b, h in slices:
        sl = (slice(b, b + 1), slice(h, h + 1))
        q, k, v, dO = (synth.to_f64(x[n][sl]) for n in ("q", "k", "v", "dO"))
        Or, Lr = attention.forward_rows(q, k, v, mode, l, c, rows)
        assert_close(f"{name} o", got["o"][sl][:, :, rows], Or)
        assert_close(f"{name} lse", got["lse"][sl][:, :, rows], Lr)
        dqr = attention.dq_rows(q, k, v, dO, mode, l, c, rows)
        assert_close(f"{name} dq", got["dq"][sl][:, :, rows], dqr)
        dkc, dvc = attention.dkv_cols(q, k, v, dO, mode, l, c, cols)
        assert_close(f"{name} dk", got["dk"][sl][:, :, cols], dkc)
        assert_close(f"{name} dv", got["dv"][sl][:, :, cols], dvc)
    # properties at every position: finite outputs, lse at least the diagonal score
    for k_ in ("o", "lse", "dq", "dk", "dv"):
        assert np.isfinite(got[k_]).all(), k_
    qd = synth.to_f64(x["q"])
    kd = synth.to_f64(x["k"])
    diag = (qd * kd).sum(-1) / np.sqrt(D)
    assert (got["lse"] >= diag - 2e-2).all()


@pytest.mark.parametrize("name", ["image32-strided", "text-fixed", "image64-strided", "image64-all",
                                  "image64-local", "image64-column",
                                  "audio-strided"])
def test_parity_full_size_sampled(cuda_device, name):
    w = synth.WORKLOADS[name]
    _sampled(name, slices=((0, 0), (w["B"] - 1, w["H"] - 1)) if w["N"] <= 3072 else ((0, 0),))


@pytest.mark.parametrize("name,sl", [("text-fixed", (0, 0)), ("text-fixed", (1, 7)),
                                     ("image64-strided", (0, 0)), ("image64-strided", (0, 15))])
def test_parity_full_size_whole_head(cuda_device, name, sl):
    """One whole (batch, head) slice of an N = 12288 workload, every element of
    O, lse, dQ, dK, dV against the oracle (the launch configuration the
    benchmark times: all heads of the workload in one call)."""
    w = synth.WORKLOADS[name]
    mode, B, H, N, D, l, c, block = (w[k] for k in ("mode", "B", "H", "N", "D", "l", "c", "block"))
    x, got, _ = run_library(mode, B, H, N, D, l, c, block)
    ref = oracle_full(x, mode, l, c, sl=sl)
    b, h = sl
    for n in ("o", "lse", "dq", "dk", "dv"):
        assert_close(f"{name} ({b},{h}) {n}", got[n][b:b + 1, h:h + 1], ref[n])


@pytest.mark.parametrize("N,l,rows,cols", [
    (1 << 18, 512, [0, 1, 777, 131071, 200000, (1 << 18) - 1], [5, 100003, (1 << 18) - 1]),
    # 2^20 positions, l = 1024: whole 128-row tiles at the start, middle and end; key columns near the end
    (1 << 20, 1024, list(range(128)) + list(range(524288, 524416)) + list(range((1 << 20) - 128, 1 << 20)),
     list(range((1 << 20) - 300, (1 << 20) - 290)) + [(1 << 20) - 1]),
])
def test_long_sequence_sampled(cuda_device, N, l, rows, cols):
    """A strided head at N = 2^18 (l = 512) and 2^20 (l = 1024): sampled rows and
    key columns against the oracle, and properties at every position."""
    mode, B, H, D, c, block = "strided", 1, 1, 64, 0, 64
    x, got, _ = run_library(mode, B, H, N, D, l, c, block)
    q, k, v, dO = (synth.to_f64(x[n]) for n in ("q", "k", "v", "dO"))
    rows = np.array(rows)
    # the oracle's rows in chunks of 16 (a row of scores at N = 2^20 is 8 MB in float64)
    parts = [rows[i:i + 16] for i in range(0, len(rows), 16)]
    Or = np.concatenate([attention.forward_rows(q, k, v, mode, l, c, p)[0] for p in parts], axis=2)
    Lr = np.concatenate([attention.forward_rows(q, k, v, mode, l, c, p)[1] for p in parts], axis=2)
    assert_close("long o", got["o"][:, :, rows], Or)
    assert_close("long lse", got["lse"][:, :, rows], Lr)
    dqr = np.concatenate([attention.dq_rows(q, k, v, dO, mode, l, c, p) for p in parts], axis=2)
    assert_close("long dq", got["dq"][:, :, rows], dqr)
    cols = np.array(cols)
    dkc, dvc = attention.dkv_cols(q, k, v, dO, mode, l, c, cols)
    assert_close("long dk", got["dk"][:, :, cols], dkc)
    assert_close("long dv", got["dv"][:, :, cols], dvc)
    for k_ in ("o", "lse", "dq", "dk", "dv"):
        assert np.isfinite(got[k_]).all(), k_


def _random_blocks(nb, seed, p=0.35):
    rng = np.random.default_rng(seed)
    rp, ci = [0], []
    for r in range(nb):
        ci += [s for s in range(r) if rng.random() < p] + [r]
        rp.append(len(ci))
    return rp, ci


@pytest.mark.parametrize("B,H,N,D,b,seed", [(1, 2, 2048, 64, 128, 0), (2, 1, 1024, 32, 256, 1),
                                            (1, 1, 1024, 128, 128, 2),
                                            # blocks smaller than a kernel tile: sub-block bits
                                            (1, 2, 2048, 64, 64, 3), (1, 1, 1024, 32, 32, 4), (2, 1, 768, 64, 16, 5),
                                            (1, 1, 1024, 128, 32, 6),
                                            (1, 1, 4096, 64, 64, 7)])  # long rows: the LONG backward shape
def test_parity_block_mask(cuda_device, B, H, N, D, b, seed):
    """A caller's block mask (sparse_attn_layout_blocks) against the oracle's BlockMask."""
    from factorized_block_sparse_b200 import sparse_attn as sa
    from oracle import patterns

    rp, ci = _random_blocks(N // b, seed)
    lay = sa.Layout.from_blocks(N, b, rp, ci)
    x, got, _ = run_library("blocks", B, H, N, D, 1, 0, b, layout=lay)
    ref = oracle_full(x, patterns.BlockMask(N, b, rp, ci), 1, 0)
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert np.isfinite(got[name]).all(), name
        assert_close(f"blocks N={N} D={D} {name}", got[name], ref[name])


@pytest.mark.parametrize("B,H,N,D,b", [(1, 2, 1024, 64, 64), (1, 1, 1024, 128, 32), (2, 1, 960, 32, 16)])
def test_parity_block_diagonal_mask(cuda_device, B, H, N, D, b):
    """A caller's mask of the diagonal blocks only (blocks below a tile): each
    64-query step meets one key tile, the case where the natural pass writes
    the final dQ itself."""
    from factorized_block_sparse_b200 import sparse_attn as sa
    from oracle import patterns

    rp, ci = _random_blocks(N // b, 0, p=0.0)
    lay = sa.Layout.from_blocks(N, b, rp, ci)
    x, got, _ = run_library("blocks", B, H, N, D, 1, 0, b, layout=lay)
    ref = oracle_full(x, patterns.BlockMask(N, b, rp, ci), 1, 0)
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert np.isfinite(got[name]).all(), name
        assert_close(f"diagonal blocks N={N} D={D} b={b} {name}", got[name], ref[name])


@pytest.mark.parametrize("mode,N,l,c,finalise,summary", [
    ("fixed", 2048, 128, 32, 0, 1),   # own block = one 128-key tile per 64-query step
    ("block", 960, 64, 0, 0, 0),
    ("fixed", 2048, 256, 32, 1, 1),   # a step of the second half of a block meets two key tiles
    ("fixed", 2048, 512, 32, 1, 0),   # natural items of 5 steps on average: the LONG shape, which adds
                                      # the summary partials itself
    ("strided", 2048, 64, 0, 1, 0),
    ("column", 2048, 64, 0, 1, 0),    # no natural view
])
def test_final_dq_pass(cuda_device, mode, N, l, c, finalise, summary):
    """The separate dQ finalise runs only where the natural view's pass cannot
    complete each dQ row with one product; the summary keys' dK/dV finalise
    only where the natural pass reduced their rows into the partials."""
    from factorized_block_sparse_b200 import sparse_attn as sa

    sa.timing_reset()
    sa.timing_enable(True)
    try:
        run_library(mode, 1, 1, N, 64, l, c, 64)
    finally:
        sa.timing_enable(False)
    kt = sa.kernel_times()
    assert kt[f"sa_bwd_finalize_dq.{mode}"][1] == finalise
    assert kt[f"sa_bwd_finalize_summary_dkv.{mode}"][1] == summary
    sa.timing_reset()


def test_block_mask_of_all_lower_blocks_equals_all(cuda_device):
    from factorized_block_sparse_b200 import sparse_attn as sa

    N, b = 1024, 128
    rp, ci = _random_blocks(N // b, 0, p=1.0)
    a = run_library("blocks", 1, 2, N, 64, 1, 0, b, layout=sa.Layout.from_blocks(N, b, rp, ci))[1]
    r = run_library("all", 1, 2, N, 64, 1, 0, b)[1]
    for name in ("o", "lse", "dk", "dv"):
        assert np.array_equal(a[name], r[name]), name

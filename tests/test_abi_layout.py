"""C ABI on the host (no GPU): the library loads, exports every symbol the
header declares, validates arguments, and its block tables are bit-exact
against the oracle's block-OR of the element masks."""

import ctypes
import json
import os
import re

import numpy as np
import pytest

from factorized_block_sparse_b200 import build, synth
from oracle import views

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sa():
    build.build()
    from factorized_block_sparse_b200 import sparse_attn

    return sparse_attn


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(sparse_attn_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(sa):
    declared = _declared_functions()
    assert declared, "no declarations found"
    assert declared == set(sa.EXPORTS)
    raw = ctypes.CDLL(sa.LIB_PATH)
    for name in declared:
        assert hasattr(raw, name), name


def test_library_has_no_libcuda_dependency(sa):
    # loads on a GPU-less host: the driver is reached through the runtime's entry-point query
    import subprocess

    out = subprocess.run(["ldd", sa.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out
    assert "libcudart.so" not in out


def test_argument_errors(sa):
    h = ctypes.c_void_p()
    L = sa.lib.sparse_attn_layout
    assert L(7, 64, 8, 0, 16, ctypes.byref(h)) == sa.SA_ERR_INVALID_ARG
    assert L(2, 64, 0, 0, 16, ctypes.byref(h)) == sa.SA_ERR_INVALID_ARG
    assert L(3, 64, 8, 0, 16, ctypes.byref(h)) == sa.SA_ERR_INVALID_ARG   # fixed needs c >= 1
    assert L(3, 64, 8, 9, 16, ctypes.byref(h)) == sa.SA_ERR_INVALID_ARG   # c <= l
    assert L(0, 64, 1, 0, 0, ctypes.byref(h)) == sa.SA_ERR_INVALID_ARG
    assert L(0, 60, 1, 0, 16, ctypes.byref(h)) == sa.SA_ERR_UNSUPPORTED   # N % block
    assert L(4, 64, 12, 0, 16, ctypes.byref(h)) == sa.SA_ERR_UNSUPPORTED  # column head: N % l
    for pat in (2, 3):                                                    # strided, fixed: any N % l
        assert L(pat, 64, 12, 4, 16, ctypes.byref(h)) == sa.SA_OK
        sa.lib.sparse_attn_layout_free(h)
    assert L(4, 64, 12, 0, 16, ctypes.byref(h)) == sa.SA_ERR_UNSUPPORTED  # column: N % l
    assert L(6, 64, 8, 0, 16, ctypes.byref(h)) == sa.SA_ERR_INVALID_ARG   # no pattern 6
    assert L(5, 64, 12, 0, 16, ctypes.byref(h)) == sa.SA_OK               # block: any l
    sa.lib.sparse_attn_layout_free(h)
    assert L(0, 64, 1, 0, 16, None) == sa.SA_ERR_INVALID_ARG
    lay = sa.Layout("strided", 256, 16, 0, 16)
    n = ctypes.c_int()
    assert sa.lib.sparse_attn_layout_export(lay.handle, 3, None, None, None, ctypes.byref(n),
                                            ctypes.byref(n)) == sa.SA_ERR_INVALID_ARG
    # compute calls reject bad arguments on the host before touching a device
    assert sa.lib.sparse_attn_fwd(None, None, None, None, None, 1, 1, 256, 32, lay.handle, None) \
        == sa.SA_ERR_INVALID_ARG
    fake = ctypes.c_void_p(4096)
    assert sa.lib.sparse_attn_fwd(fake, fake, fake, fake, fake, 1, 1, 128, 32, lay.handle, None) \
        == sa.SA_ERR_LUT
    assert sa.lib.sparse_attn_fwd(fake, fake, fake, fake, fake, 1, 1, 256, 48, lay.handle, None) \
        == sa.SA_ERR_UNSUPPORTED
    assert sa.lib.sparse_attn_fwd(fake, fake, fake, fake, fake, 0, 1, 256, 32, lay.handle, None) \
        == sa.SA_ERR_INVALID_ARG
    # an explicit softmax scale must be finite and positive (checked before any launch)
    for bad in (0.0, -0.5, float("nan"), float("inf")):
        assert sa.lib.sparse_attn_fwd_ex(fake, fake, fake, fake, fake, 1, 1, 256, 32, bad, lay.handle, None) \
            == sa.SA_ERR_INVALID_ARG
        assert sa.lib.sparse_attn_bwd_ex(*([fake] * 9), 1, 1, 256, 32, bad, lay.handle, fake, 1 << 20, None) \
            == sa.SA_ERR_INVALID_ARG
    # D = 32 rows are 64 bytes: runs of an odd number of rows cannot be moved
    # by TMA (128-byte shared-memory boundaries), so odd R or odd c > 1 is refused
    for mode, N, l, c in (("strided", 1344, 64, 0), ("column", 320, 64, 0), ("fixed", 1024, 128, 5)):
        odd = sa.Layout(mode, N, l, c, 64)
        assert sa.lib.sparse_attn_fwd(fake, fake, fake, fake, fake, 1, 1, N, 32, odd.handle, None) \
            == sa.SA_ERR_UNSUPPORTED, mode
        assert sa.lib.sparse_attn_bwd(*([fake] * 9), 1, 1, N, 32, odd.handle, fake, 1 << 30, None) \
            == sa.SA_ERR_UNSUPPORTED, mode
    assert sa.strerror(sa.SA_ERR_TIMEOUT) == "device-side wait timed out"
    assert sa.lib.sparse_attn_kernel_kinds() == 63  # 9 kernels x 7 patterns


def _compare(sa, mode, N, l, c, b, rows=None):
    lay = sa.Layout(mode, N, l, c, b)
    for v in views.views_of(mode):
        got = lay.export(v)
        ref = views.block_table(v, mode, N, l, c, b, rows=rows)
        if rows is None:
            assert got["n_rows"] == ref["n_rows"]
            assert np.array_equal(got["row_ptr"], ref["row_ptr"]), (mode, v)
            assert np.array_equal(got["col_idx"], ref["col_idx"]), (mode, v)
            assert np.array_equal(got["kind"], ref["kind"]), (mode, v)
            gt = lay.export(v, transposed=True)
            rt = views.transpose_table(ref)
            assert np.array_equal(gt["row_ptr"], rt["row_ptr"]), (mode, v, "T")
            assert np.array_equal(gt["col_idx"], rt["col_idx"]), (mode, v, "T")
            assert np.array_equal(gt["kind"], rt["kind"]), (mode, v, "T")
        else:
            rp = got["row_ptr"]
            for k, r in enumerate(rows):
                a0, a1 = rp[r], rp[r + 1]
                b0, b1 = ref["row_ptr"][k], ref["row_ptr"][k + 1]
                assert np.array_equal(got["col_idx"][a0:a1], ref["col_idx"][b0:b1]), (mode, v, r)
                assert np.array_equal(got["kind"][a0:a1], ref["kind"][b0:b1]), (mode, v, r)
    # views a pattern does not have export as empty
    for v in set(views.VIEWS) - set(views.views_of(mode)):
        assert lay.export(v)["n_rows"] == 0


@pytest.mark.parametrize("name", [n for n, w in synth.WORKLOADS.items() if w["N"] <= 12288])
def test_layout_bit_exact_named_workloads(sa, name):
    w = synth.WORKLOADS[name]
    _compare(sa, w["mode"], w["N"], w["l"], w["c"], w["block"])


def test_layout_bit_exact_audio_sampled_rows(sa):
    w = synth.WORKLOADS["audio-strided"]
    rows = [0, 1, 2, 3, 4, 5, 17, 255, 256, 511, 512, 777, 1000, 1022, 1023]
    _compare(sa, w["mode"], w["N"], w["l"], w["c"], w["block"], rows=rows)
    with open(os.path.join(ROOT, "tests", "golden", "lut_counts.json")) as f:
        gold = json.load(f)["workloads"]["audio-strided"]["views"]
    lay = sa.Layout(w["mode"], w["N"], w["l"], w["c"], w["block"])
    for v, (nf, npart) in gold.items():
        t = lay.export(v)
        assert int((t["kind"] == 0).sum()) == nf and int((t["kind"] == 1).sum()) == npart


@pytest.mark.parametrize("mode,N,l,c,b", [
    ("all", 64, 1, 0, 1), ("all", 96, 1, 0, 32), ("all", 128, 1, 0, 128),
    ("local", 128, 1, 0, 16), ("local", 128, 200, 0, 16), ("local", 120, 7, 0, 8),
    ("strided", 128, 1, 0, 16), ("strided", 128, 128, 0, 16), ("strided", 144, 12, 0, 8),
    ("strided", 64, 8, 0, 3 * 0 + 4), ("strided", 96, 6, 0, 48),
    ("fixed", 128, 16, 16, 16), ("fixed", 128, 16, 1, 8), ("fixed", 144, 12, 5, 16),
    ("fixed", 96, 24, 3, 48), ("fixed", 64, 64, 8, 16),
    # N not a multiple of l: a partial last block, with and without summary offsets of its own
    ("fixed", 136, 16, 4, 8), ("fixed", 140, 16, 6, 4), ("fixed", 1136, 128, 32, 16), ("fixed", 100, 24, 24, 4),
    ("strided", 100, 12, 0, 4), ("strided", 130, 16, 0, 2), ("strided", 1000, 64, 0, 8), ("strided", 40, 64, 0, 8),
    ("strided", 1216, 96, 0, 64), ("fixed", 40, 64, 8, 4), ("fixed", 200, 256, 64, 8),
    ("column", 128, 16, 0, 16), ("column", 144, 12, 0, 8), ("column", 128, 1, 0, 16),
    ("column", 128, 128, 0, 16), ("column", 96, 6, 0, 48),
    ("block", 128, 16, 0, 16), ("block", 120, 7, 0, 8), ("block", 64, 64, 0, 16), ("block", 96, 1, 0, 8),
])
def test_layout_bit_exact_degenerate_and_ragged(sa, mode, N, l, c, b):
    _compare(sa, mode, N, l, c, b)


def _random_blocks(nb, seed, p=0.35):
    rng = np.random.default_rng(seed)
    rp, ci = [0], []
    for r in range(nb):
        ci += [s for s in range(r) if rng.random() < p] + [r]
        rp.append(len(ci))
    return rp, ci


@pytest.mark.parametrize("N,b,seed", [(1024, 128, 0), (2048, 256, 1), (1536, 128, 2), (1024, 64, 3), (512, 32, 4),
                                      (256, 16, 5)])
def test_layout_blocks_bit_exact(sa, N, b, seed):
    from oracle import patterns

    rp, ci = _random_blocks(N // b, seed)
    lay = sa.Layout.from_blocks(N, b, rp, ci)
    bm = patterns.BlockMask(N, b, rp, ci)
    got, ref = lay.export("N"), views.block_table("N", bm, N, 1, 0, b)
    for k in ("row_ptr", "col_idx", "kind"):
        assert np.array_equal(got[k], ref[k]), k
    gt, rt = lay.export("N", transposed=True), views.transpose_table(ref)
    for k in ("row_ptr", "col_idx", "kind"):
        assert np.array_equal(gt[k], rt[k]), k
    assert lay.export("T")["n_rows"] == 0 and lay.export("S")["n_rows"] == 0


def test_layout_blocks_errors(sa):
    with pytest.raises(sa.SparseAttnError) as e:
        sa.Layout.from_blocks(256, 128, [0, 1, 2], [0, 0])          # row 1 without its diagonal
    assert e.value.status == sa.SA_ERR_INVALID_ARG
    with pytest.raises(sa.SparseAttnError) as e:
        sa.Layout.from_blocks(384, 128, [0, 1, 3, 5], [0, 1, 0, 0, 2])  # unsorted row 1
    assert e.value.status == sa.SA_ERR_INVALID_ARG
    with pytest.raises(sa.SparseAttnError) as e:
        sa.Layout.from_blocks(288, 48, [0, 1, 3, 4, 6, 7, 8], [0, 0, 1, 2, 2, 3, 4, 5])  # block 48: not supported
    assert e.value.status == sa.SA_ERR_UNSUPPORTED
    with pytest.raises(sa.SparseAttnError) as e:
        sa.Layout.from_blocks(300, 128, [0, 1, 3], [0, 0, 1])        # N % block
    assert e.value.status == sa.SA_ERR_UNSUPPORTED
    h = ctypes.c_void_p()
    assert sa.lib.sparse_attn_layout(6, 256, 1, 0, 128, ctypes.byref(h)) == sa.SA_ERR_INVALID_ARG


def test_noalloc_scratch_size_matches_header(sa):
    # the binding's copy of SA_NOALLOC_SCRATCH_BYTES must follow the header's macro
    text = open(os.path.join(ROOT, "include", "sparse_attn.h")).read()
    m = re.search(r"#define\s+SA_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*\*\s*(\d+)u\s*\*\s*(\d+)u\)", text)
    assert m, "SA_NOALLOC_SCRATCH_BYTES not found in the header"
    assert int(m.group(1)) * int(m.group(2)) * int(m.group(3)) == sa.NOALLOC_SCRATCH_BYTES

"""bench.py's per-workload accounting: element counts, algorithmic bytes and
the per-workload roofline fraction (CPU only; no kernel is run)."""

import json
import pathlib
import sys

import pytest

ROOT = pathlib.Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))

import bench  # noqa: E402
from factorized_block_sparse_b200 import synth  # noqa: E402

GOLDEN = json.loads((ROOT / "tests" / "golden" / "nnz_counts.json").read_text())["workloads"]


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
def test_element_counts_equal_the_golden_closed_forms(name):
    assert bench.element_nnz(synth.WORKLOADS[name]) == GOLDEN[name]["nnz_per_head"]


def test_algorithmic_bytes():
    w = synth.WORKLOADS["text-fixed"]
    rows = w["B"] * w["H"] * w["N"]
    assert bench.algorithmic_bytes(w) == rows * ((8 * 64 + 4) + (16 * 64 + 4))
    ws = synth.WORKLOADS["image64-strided"]
    rows_s = ws["B"] * ws["H"] * ws["N"]
    assert bench.algorithmic_bytes(ws) == rows_s * ((8 * 64 + 4) + (16 * 64 + 4) + (4 * 64 + 8))


def test_workload_lines_split_kernel_times_by_pattern():
    pk = dict(bf16=1000.0, hbm=5000.0)
    state = [dict(w=synth.WORKLOADS["text-fixed"], name="text-fixed", flops=2e11),
             dict(w=synth.WORKLOADS["image64-strided"], name="image64-strided", flops=5e10)]
    # (total ms, launches) per kernel kind, two launches each
    kt = {"sa_fwd_natural_view.fixed": (0.4, 2), "sa_bwd_natural_view.fixed": (1.0, 2),
          "sa_fwd_column_view.strided": (0.2, 2), "sa_bwd_secondary_view.strided": (0.6, 2)}
    out = bench.workload_lines(state, kt, pk)
    f = out["text-fixed"]
    assert f["fwd_ms"] == pytest.approx(0.2) and f["bwd_ms"] == pytest.approx(0.5)
    assert f["nonzero_block_tflops"] == pytest.approx(2e11 / 0.7e-3 / 1e12, rel=1e-3)
    assert f["roofline"]["bound"] == "tensor"
    assert f["roofline"]["frac"] == pytest.approx((2e11 / 1e15 * 1e3) / 0.7, rel=1e-3)
    s = out["image64-strided"]
    assert s["fwd_ms"] == pytest.approx(0.1) and s["bwd_ms"] == pytest.approx(0.3)
    # two workloads of one pattern cannot be told apart by kernel name
    assert bench.workload_lines(state + [dict(state[0])], kt, pk) is None

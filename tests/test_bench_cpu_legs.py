"""The benchmark's CPU-oracle legs run on the host alone: they must produce their record
(never fail the benchmark line) on a small workload. No GPU is used."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_backward_oracle_leg_on_the_tiny_workload(orc):
    w = bench.workload("tiny")
    rec = bench.cpu_baseline_backward(w, w.budget_blocks(w.budgets[0]), n_items=2)
    assert rec["kind"] == "oracle" and rec["extrapolated"] is True and rec["cores"] == 1
    assert rec["value"] > 0 and rec["est_s"] > 0
    assert "kept (query block, key block) pairs" in rec["sample"]

"""Host logic of bench.py: the roofline's algorithmic bytes, counted by hand on a tiny case."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_algorithmic_bytes_by_hand():
    # one sequence of 40 tokens (3 pages), 4 q-heads / 2 kv-heads
    seq_lens = np.array([40])
    sel = np.full((1, 4, 2), -1)
    cnt = np.array([[1, 2, 2, 1]])
    sel[0, 0, :1] = [0]
    sel[0, 1, :2] = [0, 2]          # group 0 union of pages: {0, 2}
    sel[0, 2, :2] = [1, 2]
    sel[0, 3, :1] = [1]             # group 1 union: {1, 2}
    union_count = np.array([[5, 7]])
    total, parts = bench.algorithmic_bytes(None, seq_lens, 4, 2, sel, cnt, union_count)
    assert parts["bounds"] == 3 * 2 * 512
    assert parts["page_table"] == 3 * 4
    assert parts["int4"] == (2 + 2) * 1088
    assert parts["kv"] == (5 + 7) * 512
    assert parts["q_o"] == 4 * (256 + 516) + 4
    assert total == sum(parts.values())


def test_traffic_only_for_matching_sources(tmp_path, monkeypatch):
    assert bench.measured_traffic() in (None,) or isinstance(bench.measured_traffic(), int)
    monkeypatch.setattr(bench, "source_hash", lambda kernel="decode_step": "not-the-sources")
    assert bench.measured_traffic() is None
    assert bench.measured_traffic("prune_rows", "dram_bytes_per_launch_n131072") is None


def test_prune_rows_bytes_by_hand():
    # 3 rows of 8 weights: 4 B per weight read, m and the count written (8 B per row), 4 B per
    # kept index when the indices are written
    assert bench.prune_rows_bytes(8, 3, 5, False) == 3 * (32 + 8)
    assert bench.prune_rows_bytes(8, 3, 5, True) == 3 * (32 + 8) + 20

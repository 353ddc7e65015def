"""Host-side helpers of bench.py: ablation list builders and the traffic lookup (CPU)."""
import json
import os

import pytest
import torch

import bench


def test_ascending_order_keeps_sets_and_padding():
    order = torch.tensor([[[5, 1, 3, -1], [2, 0, -1, -1], [7, -1, -1, -1]]], dtype=torch.int32)
    asc = bench.ascending_order(order)
    assert asc.tolist() == [[[1, 3, 5, -1], [0, 2, -1, -1], [7, -1, -1, -1]]]


def test_masked_full_lists_marks_exactly_the_selected_blocks():
    # two sequences: 300 tokens (3 blocks of 128) and 200 tokens (2 blocks)
    order = torch.tensor([[[0, -1, -1], [1, 0, -1], [2, 0, -1], [0, -1, -1], [1, -1, -1]],
                          [[0, -1, -1], [0, -1, -1], [1, 2, -1], [0, -1, -1], [0, 1, -1]]], dtype=torch.int32)
    count = torch.tensor([[1, 2, 2, 1, 1], [1, 1, 2, 1, 2]], dtype=torch.int32)
    full, cnt, keep, kmax_full = bench.masked_full_lists(order, count, [300, 200], 128)
    assert kmax_full == 3
    assert cnt.tolist() == [[1, 2, 3, 1, 2]] * 2
    for h in range(2):
        for I in range(5):
            n = int(cnt[h, I])
            assert full[h, I, :n].tolist() == list(range(n))
            assert all(x == -1 for x in full[h, I, n:].tolist())
            sel = set(order[h, I, :int(count[h, I])].tolist())
            assert {t for t in range(n) if keep[h, I, t]} == sel
            assert int(keep[h, I, n:].sum()) == 0


def test_traffic_is_reported_only_for_matching_sources(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    import hashlib
    rec = {"source_files": ["k.cu"], "source_sha256": hashlib.sha256(b"kernel v1").hexdigest(),
           "dram_read_bytes_per_launch": 100, "dram_write_bytes_per_launch": 20}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "osk_traffic_llama8b_128k.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic() == 120
    src.write_text("kernel v2")
    assert bench.measured_traffic() is None


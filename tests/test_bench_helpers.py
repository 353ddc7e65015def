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



class _FakeEvent:
    def __init__(self, **kw):
        pass

    def record(self, stream=None):
        pass

    def elapsed_time(self, other):
        return 1.0


def _fake_library(calls):
    """A stand-in for the library with the binding's signatures: it checks the
    shapes bench.py passes and records the calls (no kernels run)."""
    import types
    import block_sparse_long_14_b200 as real

    def lists(batch, kmax, out):
        H, N = batch.num_q_heads, batch.total_qblocks
        return out or dict(order=torch.zeros((H, N, kmax), dtype=torch.int32),
                           count=torch.ones((H, N), dtype=torch.int32),
                           n_hrm=torch.ones((H, N), dtype=torch.int32),
                           hrm=torch.zeros((H, N, kmax), dtype=torch.uint8))

    def proxy_top_p(batch, q, k_pages, page_table, p, kmax, ws, out=None):
        assert q.shape[0] == batch.total_tokens and 0 < p <= 1
        calls.append(("proxy_top_p", p, kmax))
        return lists(batch, kmax, out)

    def proxy(batch, q, k_pages, page_table, budget, kmax, ws, out=None):
        assert q.shape[0] == batch.total_tokens
        calls.append(("proxy", budget, kmax, batch.total_qblocks))
        return lists(batch, kmax, out)

    def attn_entry(name):
        def f(batch, q, k_pages, v_pages, page_table, order, count, kmax, thr, ws, out=None):
            assert q.shape[0] == batch.total_tokens
            assert order.shape == (batch.num_q_heads, batch.total_qblocks, kmax)
            calls.append((name, thr))
            H, N = batch.num_q_heads, batch.total_qblocks
            return out or dict(out=torch.empty_like(q), visited=torch.full((H, N), 4, dtype=torch.int32),
                               skipped=torch.ones((H, N), dtype=torch.int32))
        return f

    def alloc_workspace(batch, budget):
        nkb = (max(batch.seqlens) + batch.block_size - 1) // batch.block_size
        return torch.zeros(256, dtype=torch.uint8), (nkb if budget == 1.0 else 3)

    return types.SimpleNamespace(
        Batch=lambda *a, **k: real.Batch(*a, **{**k, "device": "cpu"}), alloc_workspace=alloc_workspace,
        proxy=proxy, proxy_top_p=proxy_top_p, attn=attn_entry("attn"), attn_delta=attn_entry("attn_delta"),
        check=lambda ws: None)


def test_pages_rules_and_cached_prefix_legs(monkeypatch):
    """The bench's informational legs call the library with consistent shapes:
    Top-p lists sized for every candidate, then tau_s = delta / N; and a
    cached-prefix batch whose Q holds each sequence's last half."""
    import numpy as np
    import block_sparse_long_14_b200 as real
    from synth import make_custom

    monkeypatch.setattr(torch.cuda, "Event", _FakeEvent)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)
    calls = []
    lib = _fake_library(calls)
    w = make_custom([1000, 300], 8, 2, 128, 128, 64, structure="llama", seed=3)

    def bf16(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)

    d = dict(q=bf16(w.q), k_pages=bf16(w.k_pages), v_pages=bf16(w.v_pages), page_table=torch.from_numpy(w.page_table))
    batch = real.Batch(w.seqlens, 8, 2, 128, 128, 64, w.num_pages, w.max_pages_per_seq, device="cpu")
    r = bench.pages_rules(lib, batch, d, 100, 1.0, None)
    assert r["p"] == bench.TOP_P and r["delta"] == bench.DELTA and r["ms"] == 1.0
    assert ("proxy_top_p", bench.TOP_P, 8) in calls and ("attn_delta", bench.DELTA) in calls
    calls.clear()
    r = bench.cached_prefix(lib, w, d, 0.1, None)
    assert (r["q_tokens"], r["kv_tokens"]) == (500 + 150, 1300)
    # present q-blocks: 8 - 500 // 128 = 5 and 3 - 150 // 128 = 2
    assert ("proxy", 0.1, 3, 7) in calls and ("attn", bench.TAU) in calls

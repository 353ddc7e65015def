"""Pins for prefill after a cached prefix (q_len < kv_len) in the oracle.

Reading (the pages of "CoSA: Accelerating Long-Context Inference via
Proxy-Kernel Co-Designed Sparse Attention" treat full prefill only): the
last Lq_s of a sequence's L_s tokens are the queries; q-blocks stay on the kv
block grid, so the first present q-block may lack its leading rows, and the
q-blocks wholly inside the prefix have no list row.

Expected values come from the full-prefill computation (whose rows for the
same queries must agree where the reading says they do), from torch's CPU
attention with an explicit mask, and from a loop-level brute force.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import dense, kap, osk
from oracle._bf16 import f32, gather_tokens
from oracle._layout import num_query_blocks, query_blocks
from synth import make_custom


def _prefix_q(w, q_lens):
    """The packed Q of the cached-prefix case: each sequence's last Lq rows."""
    parts, tok0 = [], 0
    for L, Lq in zip(w.seqlens, q_lens):
        parts.append(w.q[tok0 + L - Lq:tok0 + L])
        tok0 += L
    return np.concatenate(parts, axis=0)


def _full_rows(w, q_lens):
    """List rows of the full prefill that the cached-prefix case keeps."""
    rows, I = [], 0
    for L, Lq in zip(w.seqlens, q_lens):
        nb = (L + w.block_size - 1) // w.block_size
        rows += list(range(I + (L - Lq) // w.block_size, I + nb))
        I += nb
    return np.array(rows)


def test_query_blocks_closed_forms():
    assert query_blocks([300], [100], 64) == [(200, 3, 5, 0)]
    assert query_blocks([300, 128], None, 64) == [(0, 0, 5, 0), (0, 0, 2, 300)]
    assert query_blocks([300, 128], [1, 128], 64) == [(299, 4, 5, 0), (0, 0, 2, 1)]
    assert num_query_blocks([300, 128, 64], [100, 65, 64], 64) == 2 + 2 + 1
    for bad in ([0], [301], [-1]):
        with pytest.raises(ValueError):
            query_blocks([300], bad, 64)


@pytest.fixture(scope="module")
def wl():
    # kv lengths with ragged tails; d = 64 keeps the oracle fast
    return make_custom([5 * 64 + 37, 3 * 64, 2 * 64 + 5], 4, 2, 64, 64, 16, structure="llama", seed=21)


ALIGNED = [64 * 2 + 37, 64 * 2, 64 * 2 + 5]          # prefixes 3 * 64, 64, 0
UNALIGNED = [100, 3 * 64 - 104, 1]                  # prefixes 257 (mid-block), 104 (two whole sub-rows absent), 132


def test_dense_prefix_matches_torch_masked_attention(wl):
    q_lens = UNALIGNED
    qp = _prefix_q(wl, q_lens)
    out = dense.dense_causal(qp, wl.k_pages, wl.v_pages, wl.page_table, wl.seqlens, 2, q_lens=q_lens)
    tq0 = 0
    for s, (L, Lq) in enumerate(zip(wl.seqlens, q_lens)):
        off = L - Lq
        K = f32(gather_tokens(wl.k_pages, wl.page_table[s], L)).astype(np.float64)
        V = f32(gather_tokens(wl.v_pages, wl.page_table[s], L)).astype(np.float64)
        Q = f32(qp[tq0:tq0 + Lq]).astype(np.float64)
        mask = torch.arange(L)[None, :] <= (off + torch.arange(Lq))[:, None]      # [Lq, L]
        for h in range(4):
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(Q[:, h])[None], torch.from_numpy(K[:, h // 2])[None],
                torch.from_numpy(V[:, h // 2])[None], attn_mask=mask[None])[0].numpy()
            np.testing.assert_allclose(out[tq0:tq0 + Lq, h], ref, rtol=0, atol=1e-12)
        tq0 += Lq


def test_dense_prefix_rows_equal_full_prefill_rows(wl):
    q_lens = UNALIGNED
    full = dense.dense_causal(wl.q, wl.k_pages, wl.v_pages, wl.page_table, wl.seqlens, 2)
    part = dense.dense_causal(_prefix_q(wl, q_lens), wl.k_pages, wl.v_pages, wl.page_table,
                              wl.seqlens, 2, q_lens=q_lens)
    np.testing.assert_allclose(part, _prefix_q_f64(full, wl.seqlens, q_lens), rtol=0, atol=1e-12)


def _prefix_q_f64(x, seqlens, q_lens):
    parts, tok0 = [], 0
    for L, Lq in zip(seqlens, q_lens):
        parts.append(x[tok0 + L - Lq:tok0 + L])
        tok0 += L
    return np.concatenate(parts, axis=0)


@pytest.mark.parametrize("budget", [0.3, 1.0])
def test_kap_aligned_prefix_lists_equal_full_prefill_rows(wl, budget):
    """With the prefix on the block grid every present q-block is whole, so
    its list is the full prefill's list for that q-block, bit for bit."""
    q_lens = ALIGNED
    full = kap.kap_proxy(wl.q, wl.k_pages, wl.page_table, wl.seqlens, 2, 64, budget)
    part = kap.kap_proxy(_prefix_q(wl, q_lens), wl.k_pages, wl.page_table, wl.seqlens, 2, 64, budget,
                         q_lens=q_lens)
    rows = _full_rows(wl, q_lens)
    assert part["count"].shape[1] == len(rows) == num_query_blocks(wl.seqlens, q_lens, 64)
    for key in ("order", "count", "n_hrm", "hrm"):
        assert np.array_equal(part[key], full[key][:, rows]), key


def test_kap_unaligned_prefix_brute_force(wl):
    """Loop-level restatement: pooled sums over the present rows only, one
    fp32 add at a time; sub-rows with no present row take no part in HRM."""
    q_lens = UNALIGNED
    b, g, budget = 64, 16, 0.4
    qp = _prefix_q(wl, q_lens)
    r = kap.kap_proxy(qp, wl.k_pages, wl.page_table, wl.seqlens, 2, b, budget, q_lens=q_lens)
    bp = kap.budget_bp(budget)
    I, tq0 = 0, 0
    for s, (L, Lq) in enumerate(zip(wl.seqlens, q_lens)):
        off = L - Lq
        k8, ks = kap.quantize_keys(*kap.pool_keys(f32(gather_tokens(wl.k_pages, wl.page_table[s], L)), L, b))
        Q = f32(qp[tq0:tq0 + Lq])
        nb = (L + b - 1) // b
        for i in range(off // b, nb):
            for h in range(4):
                kv = h // 2
                subs, valid = [], []
                for rr in range(b // g):
                    acc = np.zeros(64, dtype=np.float32)
                    present = False
                    for pos in range(i * b + rr * g, i * b + (rr + 1) * g):
                        if off <= pos < L:
                            acc = (acc + Q[pos - off, h]).astype(np.float32)
                            present = True
                    subs.append(acc)
                    valid.append(present)
                blk = np.zeros(64, dtype=np.float32)
                for v in subs:
                    blk = (blk + v).astype(np.float32)

                def score(vec, j):
                    q8 = kap.quantize_int8(vec)[0].astype(np.int64)
                    dot = int(sum(int(a) * int(c) for a, c in zip(q8, k8[j, kv].astype(np.int64))))
                    return float(np.float32(np.float32(dot) * ks[j, kv]))

                n = i + 1
                sc = [score(blk, j) for j in range(n)]
                hrm = set()
                for rr in range(b // g):
                    if valid[rr]:
                        vals = [score(subs[rr], j) for j in range(n)]
                        hrm.add(max(range(n), key=lambda j: (vals[j], -j)))
                ranked = sorted(range(n), key=lambda j: (j not in hrm, -sc[j], j))
                k_i = max(1, -(-n * bp // 10000))
                row = I + i - off // b
                assert r["count"][h, row] == k_i
                assert r["order"][h, row, :k_i].tolist() == ranked[:k_i]
                assert r["hrm"][h, row, :k_i].tolist() == [int(j in hrm) for j in ranked[:k_i]]
        I += nb - off // b
        tq0 += Lq


@pytest.mark.parametrize("q_lens", [ALIGNED, UNALIGNED])
def test_osk_prefix_full_budget_reduces_to_dense(wl, q_lens):
    qp = _prefix_q(wl, q_lens)
    r = kap.kap_proxy(qp, wl.k_pages, wl.page_table, wl.seqlens, 2, 64, 1.0, q_lens=q_lens)
    o = osk.osk(qp, wl.k_pages, wl.v_pages, wl.page_table, wl.seqlens, 2, 64, r["order"], r["count"],
                0.0, q_lens=q_lens)
    ref = dense.dense_causal(qp, wl.k_pages, wl.v_pages, wl.page_table, wl.seqlens, 2, q_lens=q_lens)
    assert not np.isnan(o["out"]).any()
    np.testing.assert_allclose(o["out"], ref, rtol=0, atol=1e-10)
    assert np.all(o["skipped"] == 0)


def test_osk_aligned_prefix_tiles_equal_full_prefill_tiles(wl):
    """Same lists, same whole tiles: outputs, skip sets and deltas agree with
    the full prefill's, with the in-kernel skip active."""
    q_lens = ALIGNED
    tau = 2e-2
    full = kap.kap_proxy(wl.q, wl.k_pages, wl.page_table, wl.seqlens, 2, 64, 0.5)
    of = osk.osk(wl.q, wl.k_pages, wl.v_pages, wl.page_table, wl.seqlens, 2, 64, full["order"],
                 full["count"], tau)
    rows = _full_rows(wl, q_lens)
    qp = _prefix_q(wl, q_lens)
    op = osk.osk(qp, wl.k_pages, wl.v_pages, wl.page_table, wl.seqlens, 2, 64, full["order"][:, rows],
                 full["count"][:, rows], tau, q_lens=q_lens)
    assert of["skipped"][:, rows].sum() > 0                 # the skip path is exercised
    for key in ("visited", "skipped", "skip"):
        assert np.array_equal(op[key], of[key][:, rows]), key
    np.testing.assert_array_equal(op["delta"], of["delta"][:, rows])
    np.testing.assert_allclose(op["out"], _prefix_q_f64(of["out"], wl.seqlens, q_lens), rtol=0, atol=1e-12)


def test_remap_prefix_rows_equal_full_prefill_rows(wl):
    q_lens = UNALIGNED
    full = kap.kap_proxy(wl.q, wl.k_pages, wl.page_table, wl.seqlens, 2, 64, 0.5)
    rows = _full_rows(wl, q_lens)
    pf = kap.remap(full["order"], full["count"], wl.page_table, wl.seqlens, 64, 16)
    pp = kap.remap(full["order"][:, rows], full["count"][:, rows], wl.page_table, wl.seqlens, 64, 16,
                   q_lens=q_lens)
    assert np.array_equal(pp, pf[:, rows])


def test_top_p_counts_only_present_rows():
    """The Top-p mean logit divides by the q-block's present rows: with a
    constant query the mean logit, hence the cut, is the same whatever the
    prefix (two-block construction: z_0 = 2 exactly, share 64e^2/(64e^2+32))."""
    from synth import from_arrays
    L, b, d = 96, 64, 64
    q = np.full((L, 1, d), 0.5, dtype=np.float32)
    k = np.full((L, 1, d), 0.5, dtype=np.float32)
    k[b:, 0, d // 2:] = -0.5
    w = from_arrays([q], [k], [np.ones((L, 1, d), dtype=np.float32)], b, 32, shuffle=True, seed=5)
    share0 = 64 * math.exp(2.0) / (64 * math.exp(2.0) + 32)
    for Lq in (96, 32, 16, 5):
        qp = _prefix_q(w, [Lq])
        for p, want in ((share0 - 1e-3, 1), (share0 + 1e-3, 2)):
            r = kap.kap_proxy_top_p(qp, w.k_pages, w.page_table, w.seqlens, 1, b, p, q_lens=[Lq])
            assert r["count"][0, -1] == want, (Lq, p)


def test_absent_sub_rows_take_no_part_in_hrm():
    """L = 192, b = 64, prefix 104: q-block 1 keeps rows 104..127, so its
    sub-rows 0 and 1 are wholly absent.  Queries point along +e0, key block 0
    along -e0 and key block 1 along +e0: every present sub-row's argmax is
    block 1, so block 0 must not be HRM.  (An absent sub-row counted as valid
    would score 0 everywhere and flag block 0, the lowest index.)"""
    from synth import from_arrays
    L, b, d = 192, 64, 16
    q = np.zeros((L, 1, d), dtype=np.float32)
    q[:, 0, 0] = 1.0
    k = np.zeros((L, 1, d), dtype=np.float32)
    k[:b, 0, 0] = -1.0
    k[b:2 * b, 0, 0] = 1.0
    k[2 * b:, 0, 1] = 1.0
    w = from_arrays([q], [k], [np.ones((L, 1, d), dtype=np.float32)], b, 32, shuffle=True, seed=9)
    qp = _prefix_q(w, [L - 104])
    r = kap.kap_proxy(qp, w.k_pages, w.page_table, w.seqlens, 1, b, 1.0, q_lens=[L - 104])
    assert r["count"][0].tolist() == [2, 3]                  # q-blocks 1 and 2 are present
    assert r["order"][0, 0, :2].tolist() == [1, 0]
    assert r["hrm"][0, 0, :2].tolist() == [1, 0]
    assert r["n_hrm"][0, 0] == 1

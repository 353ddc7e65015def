"""Pins for the OSK, dense and remap oracles (CPU only).

"CoSA ...": §3.1 dense attention (the closed form the OSK must reduce to at
budget 100% and tau = 0); §3.2 order invariance of online softmax (P2);
§3.3 the skip's two limitations -- the running max is not the global max
(L2.1) and the per-row AND lets one row veto (L2.2); §4.3 the tile-wide vote
and any-order page visiting.
"""

import math

import numpy as np
import pytest
import torch

from oracle import dense, kap, osk
from synth import from_arrays, make_custom, make_workload


def _dense_torch(w):
    """Dense causal attention via torch's CPU fp64 SDPA (a library routine)."""
    from oracle._bf16 import f32, gather_tokens
    G = w.num_q_heads // w.num_kv_heads
    outs, tok0 = [], 0
    for s, L in enumerate(w.seqlens):
        q = torch.from_numpy(f32(w.q[tok0:tok0 + L]).astype(np.float64)).transpose(0, 1)
        k = torch.from_numpy(f32(gather_tokens(w.k_pages, w.page_table[s], L)).astype(np.float64))
        v = torch.from_numpy(f32(gather_tokens(w.v_pages, w.page_table[s], L)).astype(np.float64))
        k = k.transpose(0, 1).repeat_interleave(G, dim=0)
        v = v.transpose(0, 1).repeat_interleave(G, dim=0)
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
        outs.append(o.transpose(0, 1).numpy())
        tok0 += L
    return np.concatenate(outs, axis=0)


@pytest.mark.parametrize("case", ["tiny", "ragged_paged"])
def test_dense_oracle_matches_library_sdpa(case):
    w = make_workload(1) if case == "tiny" else make_custom([333, 70, 256], 4, 2, 32, 64, 16,
                                                             structure="random", seed=2)
    ref = _dense_torch(w)
    got = dense.dense_causal(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads)
    assert np.abs(ref - got).max() < 1e-12


@pytest.mark.parametrize("case", ["tiny", "ragged_paged"])
def test_full_budget_no_skip_equals_dense(case):
    w = make_workload(1) if case == "tiny" else make_custom([333, 70, 256], 4, 2, 32, 64, 16,
                                                             structure="llama", seed=3)
    r = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, 1.0)
    o = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size,
                r["order"], r["count"], 0.0)
    ref = dense.dense_causal(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads)
    assert np.abs(o["out"] - ref).max() < 1e-12
    assert (o["skipped"] == 0).all()


def test_order_invariance_without_skip():
    """P2: with tau = 0 the visit order does not change the output."""
    w = make_custom([700, 200], 4, 2, 64, 64, 32, structure="llama", seed=4)
    r = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, 2, w.block_size, 0.4)
    a = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, 2, w.block_size,
                r["order"], r["count"], 0.0)
    rng = np.random.default_rng(0)
    perm = r["order"].copy()
    for h in range(perm.shape[0]):
        for I in range(perm.shape[1]):
            c = r["count"][h, I]
            perm[h, I, :c] = rng.permutation(perm[h, I, :c])
    b = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, 2, w.block_size,
                perm, r["count"], 0.0)
    assert np.abs(a["out"] - b["out"]).max() < 1e-12


# ------------------------------------------------- skip rule, constructed

def _two_block_tile(d=16, b=16, low=-20.0, outlier_row=None):
    """Query rows all e0; key block A logits 0, key block B logits `low` per row.

    Keys at positions 0..2b-1, queries at positions >= 2b (all keys visible).
    """
    rng = np.random.default_rng(7)
    q = np.zeros((b, d))
    q[:, 0] = 1.0
    scale = 1.0 / math.sqrt(d)
    KA = np.zeros((b, d))
    KB = np.zeros((b, d))
    KB[:, 0] = low / scale
    if outlier_row is not None:
        q[outlier_row, 1] = 1.0
        KB[:, 1] = -low / scale          # that row sees logit 0 in block B too
    VA = rng.standard_normal((b, d))
    VB = rng.standard_normal((b, d))
    blocks = {0: (KA, VA, np.arange(0, b)), 1: (KB, VB, np.arange(b, 2 * b))}
    return q, np.arange(2 * b, 3 * b), (lambda j: blocks[j]), scale, VA, VB


def test_skip_when_running_max_already_high():
    q, qpos, blocks, scale, VA, VB = _two_block_tile()
    out, skipped, delta = osk.osk_tile(q, qpos, blocks, [0, 1], 1e-4, scale)
    assert skipped.tolist() == [False, True]
    assert delta[1] == pytest.approx(-20.0)
    # block A alone: uniform weights over its keys
    assert np.abs(out - VA.mean(axis=0)[None, :]).max() < 1e-12


def test_running_max_is_not_global_max():
    """L2.1: visiting the negligible block first, it cannot be skipped."""
    q, qpos, blocks, scale, VA, VB = _two_block_tile()
    out, skipped, _ = osk.osk_tile(q, qpos, blocks, [1, 0], 1e-4, scale)
    assert skipped.tolist() == [False, False]
    w_b = math.exp(-20.0)
    expect = (VA.sum(0) + w_b * VB.sum(0)) / (16 + 16 * w_b)
    assert np.abs(out - expect[None, :]).max() < 1e-12


def test_one_row_vetoes_the_tile_skip():
    """L2.2 (bucket effect): one row for which block B matters keeps it for the whole tile."""
    q, qpos, blocks, scale, VA, VB = _two_block_tile(outlier_row=5)
    out, skipped, delta = osk.osk_tile(q, qpos, blocks, [0, 1], 1e-4, scale)
    assert skipped.tolist() == [False, False]
    assert delta[1] == pytest.approx(0.0, abs=1e-12)
    ref_rows = np.delete(np.arange(16), 5)
    w_b = math.exp(-20.0)
    expect = (VA.sum(0) + w_b * VB.sum(0)) / (16 + 16 * w_b)
    assert np.abs(out[ref_rows] - expect[None, :]).max() < 1e-12
    assert np.abs(out[5] - (VA.sum(0) + VB.sum(0)) / 32).max() < 1e-12


def test_threshold_edges():
    q, qpos, blocks, scale, *_ = _two_block_tile(low=-20.0)
    # tau = 0 never skips; ln(tau) just below / above delta flips the decision
    assert not osk.osk_tile(q, qpos, blocks, [0, 1], 0.0, scale)[1].any()
    assert osk.osk_tile(q, qpos, blocks, [0, 1], math.exp(-19.99), scale)[1].tolist() == [False, True]
    assert osk.osk_tile(q, qpos, blocks, [0, 1], math.exp(-20.01), scale)[1].tolist() == [False, False]
    # the first visited block is never skipped, even with tau close to 1
    assert osk.osk_tile(q, qpos, blocks, [1, 0], 0.999, scale)[1][0] == False  # noqa: E712


def test_tau_at_or_above_one_follows_the_rule_as_written():
    """tau = delta / L can exceed 1 for a sequence shorter than delta.  The rule
    stays "skip iff delta < ln tau": a block whose logits sit 0.5 above the
    running max is skipped at tau = 2 (ln 2 = 0.69) and kept at tau = 1.5
    (ln 1.5 = 0.41); a skipped block changes neither m nor l nor O."""
    q, qpos, blocks, scale, VA, VB = _two_block_tile(low=0.5)
    out, skipped, delta = osk.osk_tile(q, qpos, blocks, [0, 1], 2.0, scale)
    assert skipped.tolist() == [False, True]
    assert delta[1] == pytest.approx(0.5)
    assert np.abs(out - VA.mean(axis=0)[None, :]).max() < 1e-12
    out, skipped, _ = osk.osk_tile(q, qpos, blocks, [0, 1], 1.5, scale)
    assert skipped.tolist() == [False, False]
    w_b = math.exp(0.5)
    expect = (VA.sum(0) + w_b * VB.sum(0)) / (16 + 16 * w_b)
    assert np.abs(out - expect[None, :]).max() < 1e-12


@pytest.mark.parametrize("tau", [1e-4, 1e-3, 1e-2, 1e-1])
def test_skip_error_bound(tau):
    """Each skipped key weighs < tau relative to the row max, and l >= 1, so
    |O_tau - O_0| <= 2 * tau * (#keys in skipped blocks) * max|V| per row."""
    w = make_custom([1200, 500], 4, 2, 64, 64, 32, structure="llama", seed=6)
    r = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, 2, w.block_size, 1.0)
    args = (w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, 2, w.block_size, r["order"], r["count"])
    o0 = osk.osk(*args, 0.0)
    ot = osk.osk(*args, tau)
    from oracle._bf16 import f32
    vmax = np.abs(f32(w.v_pages)).max()
    b = w.block_size
    assert ot["skipped"].sum() > 0
    tok0, I = 0, 0
    for L in w.seqlens:
        nqb = (L + b - 1) // b
        for i in range(nqb):
            for h in range(4):
                nskip = int(ot["skip"][h, I + i].sum()) * b
                rows = slice(tok0 + i * b, tok0 + min(L, (i + 1) * b))
                err = np.abs(ot["out"][rows, h] - o0["out"][rows, h]).max()
                assert err <= 2 * tau * nskip * vmax + 1e-12
        tok0 += L
        I += nqb


# --------------------------------------------------------------------- remap

@pytest.mark.parametrize("b,b_p", [(128, 64), (64, 16), (64, 64)])
def test_remap_points_at_the_listed_blocks(b, b_p):
    """Mark every physical page with (sequence, logical page); the remapped
    list must then name, in order, the logical pages of each listed block."""
    seqlens = [3 * b + 10, b, 5 * b - 1]
    w = make_custom(seqlens, 2, 1, 64, b, b_p, structure="random", seed=8)
    P = w.k_pages.shape[0]
    ident = {}
    for s, L in enumerate(seqlens):
        for lp in range((L + b_p - 1) // b_p):
            ident[int(w.page_table[s, lp])] = (s, lp)
    assert len(ident) == P
    r = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, 1, b, 0.5)
    pages = kap.remap(r["order"], r["count"], w.page_table, seqlens, b, b_p)
    ppb = b // b_p
    assert pages.shape == (2, r["order"].shape[1], r["kmax"] * ppb)
    I = 0
    for s, L in enumerate(seqlens):
        for i in range((L + b - 1) // b):
            for h in range(2):
                c = r["count"][h, I]
                for t in range(r["kmax"]):
                    for u in range(ppb):
                        p = pages[h, I, t * ppb + u]
                        j = r["order"][h, I, t]
                        if t < c and j * b + u * b_p < L:
                            assert ident[int(p)] == (s, j * ppb + u)
                        else:
                            assert p == -1
            I += 1

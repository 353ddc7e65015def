"""Pins for the KAP oracle (CPU only).

Each test checks the oracle against something other than itself: IEEE
rounding facts, exact integer arithmetic, a hand-derived construction
(tests/golden/hrm_construction.json), the quantisation error bound, brute
force over tiny inputs, or the selection invariants the pages state
("CoSA ...", Appendix C.1: HRM group first, leading entries kept under the
budget; §4.1: stage-1 budget).
"""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import kap
from oracle._bf16 import f32, gather_tokens
from synth import from_arrays, make_custom, make_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- quantisation

def test_quantize_rounds_half_to_even():
    # M = 127 -> inv = 1 exactly, so q = rint(v): IEEE round-half-to-even.
    v = np.array([[127.0, 2.5, -2.5, 3.5, 0.5, -0.5, 1.5, -126.5]], dtype=np.float32)
    q, M = kap.quantize_int8(v)
    assert M[0] == 127.0
    assert q.tolist() == [[127, 2, -2, 4, 0, 0, 2, -126]]


def test_quantize_zero_and_subnormal_vectors():
    v = np.zeros((2, 16), dtype=np.float32)
    v[1, 3] = np.float32(1e-40)      # subnormal max
    q, _ = kap.quantize_int8(v)
    assert not q.any()
    k8, ks = kap.quantize_keys(v[:, None, :], np.array([5, 7]))
    assert not k8.any() and not ks.any()


def test_quantize_error_bound_and_extremes():
    rng = np.random.default_rng(0)
    v = (rng.standard_normal((500, 128)) * rng.uniform(1e-3, 1e3, (500, 1))).astype(np.float32)
    q, M = kap.quantize_int8(v)
    assert np.all(np.abs(q).max(axis=1) == 127)            # the max-|v| element maps to +-127
    deq = q.astype(np.float64) * (M.astype(np.float64) / 127.0)[:, None]
    # |v - q M/127| <= M/254 up to the fp32 rounding of inv and of the product
    assert np.all(np.abs(v - deq) <= (M.astype(np.float64) / 254.0)[:, None] * (1 + 1e-5))


def test_int_dots_exact():
    rng = np.random.default_rng(1)
    a = rng.integers(-127, 128, (7, 32)).astype(np.int8)
    b = rng.integers(-127, 128, (5, 32)).astype(np.int8)
    brute = [[sum(int(x) * int(y) for x, y in zip(a[i], b[j])) for j in range(5)] for i in range(7)]
    assert kap.int_dots(a, b).tolist() == brute
    ext = np.full((3, 128), 127, dtype=np.int8)
    ext[1] = -127
    assert kap.int_dots(ext, ext).tolist() == (ext.astype(np.int64) @ ext.astype(np.int64).T).tolist()
    assert abs(int(kap.int_dots(ext, ext).max())) == 127 * 127 * 128


# --------------------------------------------------------------------- pooling

def _integer_workload(seqlens, Hq, Hkv, d, b, b_p, seed):
    rng = np.random.default_rng(seed)
    qs = [rng.integers(-3, 4, (L, Hq, d)).astype(np.float32) for L in seqlens]
    ks = [rng.integers(-3, 4, (L, Hkv, d)).astype(np.float32) for L in seqlens]
    vs = [rng.standard_normal((L, Hkv, d)).astype(np.float32) for L in seqlens]
    w = from_arrays(qs, ks, vs, b, b_p, shuffle=True, seed=seed)
    # poison the tail slots of partial pages: pooling must never read them
    for s, L in enumerate(seqlens):
        n = (L + b_p - 1) // b_p
        if L % b_p:
            w.k_pages[w.page_table[s, n - 1], :, L % b_p:, :] = 0x4780   # bf16 65536.0
    return w, qs, ks


@pytest.mark.parametrize("b,b_p", [(64, 64), (64, 16), (128, 32)])
def test_pooling_matches_exact_integer_sums(b, b_p):
    seqlens = [3 * b + 37, b - 5, 2 * b]
    w, qs, ks = _integer_workload(seqlens, 4, 2, 32, b, b_p, seed=b + b_p)
    tok0 = 0
    for s, L in enumerate(seqlens):
        kf = f32(gather_tokens(w.k_pages, w.page_table[s], L))
        sums, ntok = kap.pool_keys(kf, L, b)
        nkb = (L + b - 1) // b
        for j in range(nkb):
            exact = ks[s][j * b:min(L, (j + 1) * b)].astype(np.int64).sum(axis=0)
            assert np.array_equal(sums[j].astype(np.int64), exact)
            assert ntok[j] == min(b, L - j * b)
        sub, blk, sub_valid = kap.pool_queries(f32(w.q[tok0:tok0 + L]), L, b)
        for i in range(nkb):
            rows = qs[s][i * b:min(L, (i + 1) * b)].astype(np.int64)
            assert np.array_equal(blk[i].astype(np.int64), rows.sum(axis=0))
            for r in range(b // 16):
                part = qs[s][i * b + r * 16:min(L, i * b + (r + 1) * 16)].astype(np.int64)
                assert sub_valid[i, r] == (i * b + r * 16 < L)
                assert np.array_equal(sub[i, r].astype(np.int64), part.sum(axis=0))
        tok0 += L


# ---------------------------------------------------------------------- scores

@pytest.mark.parametrize("cfg", ["tiny", "ragged"])
def test_scores_within_quantisation_bound_of_pooled_dot(cfg):
    """score_ij * (Mq_i / 127) approximates (sum of q-block rows) . (mean of key block).

    Quantisation moves each element by at most half a step, which bounds the
    error of the dot product; a dropped 1/n_tok, a wrong scale or a wrong GQA
    head mapping fails by orders of magnitude.
    """
    if cfg == "tiny":
        w = make_workload(1)
    else:
        w = make_custom([700, 300], 4, 2, 64, 64, 32, structure="random", seed=5)
    b, G = w.block_size, w.num_q_heads // w.num_kv_heads
    eps = 2.0 ** -24
    tok0 = 0
    for s, L in enumerate(w.seqlens):
        kf = f32(gather_tokens(w.k_pages, w.page_table[s], L))
        ksum, ntok = kap.pool_keys(kf, L, b)
        k8, ks = kap.quantize_keys(ksum, ntok)
        _, blk, _ = kap.pool_queries(f32(w.q[tok0:tok0 + L]), L, b)
        q8, Mq = kap.quantize_int8(blk)
        _, Mk = kap.quantize_int8(ksum)
        for h in range(w.num_q_heads):
            kv = h // G
            score = kap.scores_from_dots(kap.int_dots(q8[:, h], k8[:, kv]), ks[:, kv])
            Q = blk[:, h].astype(np.float64)                              # [nqb, d]
            Kbar = ksum[:, kv].astype(np.float64) / ntok[:, None]         # [nkb, d]
            exact = Q @ Kbar.T
            approx = score.astype(np.float64) * (Mq[:, h].astype(np.float64) / 127.0)[:, None]
            eq = Mq[:, h].astype(np.float64)[:, None] / 254.0             # [nqb, 1]
            ek = (Mk[:, kv].astype(np.float64) / (254.0 * ntok))[None, :]  # [1, nkb]
            bound = (np.abs(Q).sum(1)[:, None] * ek + eq * np.abs(Kbar).sum(1)[None, :]
                     + Q.shape[1] * eq * ek)
            bound += 4 * eps * np.abs(approx) + 1e-30
            assert np.all(np.abs(exact - approx) <= bound * (1 + 1e-6))
        tok0 += L


# ------------------------------------------------------------ HRM + ordering

def _hrm_workload():
    spec = json.load(open(os.path.join(GOLDEN, "hrm_construction.json")))
    c = spec["construction"]
    L, d, b = 384, 8, 64
    q = np.zeros((L, 1, d), dtype=np.float32)
    for r in range(4):
        q[5 * b + 16 * r:5 * b + 16 * (r + 1), 0, r] = 1.0
    k = np.zeros((L, 1, d), dtype=np.float32)
    for j in range(6):
        for dim in c["support"][str(j)]:
            k[j * b:(j + 1) * b, 0, dim] = c["a"][str(j)]
    v = np.ones((L, 1, d), dtype=np.float32)
    return from_arrays([q], [k], [v], b, 32, shuffle=True, seed=3), spec


@pytest.mark.parametrize("budget", ["1.0", "0.6", "0.3"])
def test_hrm_first_flag_grouped_order_constructed(budget):
    w, spec = _hrm_workload()
    r = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, 1, w.block_size, float(budget))
    exp = spec["expected"][f"budget_{budget}"]
    i = spec["qblock"]
    k_i = int(r["count"][0, i])
    assert k_i == len(exp["order"])
    assert r["order"][0, i, :k_i].tolist() == exp["order"]
    assert r["hrm"][0, i, :k_i].tolist() == exp["hrm"]
    assert int(r["n_hrm"][0, i]) == exp["n_hrm"]
    assert np.all(r["order"][0, i, k_i:] == -1)


def test_budget_count_formula():
    assert kap.budget_bp(0.05) == 500 and kap.budget_bp(0.1) == 1000 and kap.budget_bp(1.0) == 10000
    # k_i = max(1, ceil(n_i * budget)) exactly, for the budgets the workloads use
    for budget in (0.05, 0.1, 0.2, 0.25, 1.0):
        for n in range(1, 1025):
            assert kap.keep_count(n, kap.budget_bp(budget)) == max(1, math.ceil(n * Fraction(str(budget))))
    # 128K tokens at b = 128, 5%: 26,728 kept blocks per head, kmax 52
    assert sum(kap.keep_count(n, 500) for n in range(1, 1025)) == 26728
    assert kap.kmax_for(1024, 0.05) == 52


def _row_scores(w, s, tok0):
    b = w.block_size
    L = w.seqlens[s]
    kf = f32(gather_tokens(w.k_pages, w.page_table[s], L))
    k8, ks = kap.quantize_keys(*kap.pool_keys(kf, L, b))
    sub, blk, sub_valid = kap.pool_queries(f32(w.q[tok0:tok0 + L]), L, b)
    return k8, ks, kap.quantize_int8(sub)[0], kap.quantize_int8(blk)[0], sub_valid


@pytest.mark.parametrize("cfg,budget", [("tiny", 0.25), ("tiny", 1.0), ("ragged", 0.2)])
def test_selection_brute_force_and_invariants(cfg, budget):
    if cfg == "tiny":
        w = make_workload(1)
    else:
        w = make_custom([1100, 260, 64], 4, 2, 64, 64, 16, structure="llama", seed=11)
    r = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, budget)
    G = w.num_q_heads // w.num_kv_heads
    bp = kap.budget_bp(budget)
    tok0, I = 0, 0
    for s, L in enumerate(w.seqlens):
        k8, ks, q8s, q8b, sub_valid = _row_scores(w, s, tok0)
        nqb = (L + w.block_size - 1) // w.block_size
        for i in range(nqb):
            for h in range(w.num_q_heads):
                kv = h // G
                n = i + 1
                sc = [float(np.float32(np.float32(int(np.dot(q8b[i, h].astype(np.int64), k8[j, kv].astype(np.int64)))) * ks[j, kv])) for j in range(n)]
                hrm = set()
                for rr in range(q8s.shape[1]):
                    if not sub_valid[i, rr]:
                        continue
                    best, arg = None, None
                    for j in range(n):
                        v = float(np.float32(np.float32(int(np.dot(q8s[i, rr, h].astype(np.int64), k8[j, kv].astype(np.int64)))) * ks[j, kv]))
                        if best is None or v > best:
                            best, arg = v, j
                    hrm.add(arg)
                ranked = sorted(range(n), key=lambda j: (j not in hrm, -sc[j], j))
                k_i = max(1, -(-n * bp // 10000))
                assert r["count"][h, I + i] == k_i
                assert r["order"][h, I + i, :k_i].tolist() == ranked[:k_i]
                flags = r["hrm"][h, I + i, :k_i].tolist()
                assert flags == [int(j in hrm) for j in ranked[:k_i]]
                assert flags == sorted(flags, reverse=True)          # HRM entries form a prefix
                assert r["n_hrm"][h, I + i] == min(len(hrm), k_i) >= 1
                if budget == 1.0:
                    assert sorted(r["order"][h, I + i, :k_i].tolist()) == list(range(n))
        tok0 += L
        I += nqb


def test_planted_salient_blocks_selected():
    """Tiny workload: each planted key block is kept for the q-block it was aimed at."""
    w = make_workload(1)
    r = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, 1, w.block_size, 0.25)
    for c, i in w.meta["sequences"][0]["plants"]:
        for h in range(w.num_q_heads):
            assert c in r["order"][h, i, :r["count"][h, i]].tolist()


def test_realized_budget_tracks_request():
    w = make_workload(1)
    for budget in (0.25, 0.5, 1.0):
        r = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, 1, w.block_size, budget)
        n = np.arange(1, 17)
        realized = r["count"].sum() / (2 * n.sum())
        assert budget <= realized <= budget + 16 / n.sum()


def test_golden_tiny_orders_unchanged():
    """Regression fixture written by tests/golden/make_golden.py from the oracle."""
    g = json.load(open(os.path.join(GOLDEN, "tiny_proxy.json")))
    w = make_workload(1)
    r = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, 1, w.block_size, g["budget"])
    assert r["order"].tolist() == g["order"]
    assert r["hrm"].tolist() == g["hrm"]
    assert r["count"].tolist() == g["count"]

"""Pins for the oracle's Top-p stage-1 cut (oracle.kap.top_p_count and
kap_proxy_top_p).

The pages of "CoSA: Accelerating Long-Context Inference via Proxy-Kernel
Co-Designed Sparse Attention" give the Top-p values they run with (§5.1
"Hyperparameters"; Appendix D.1) but not the mass being cut.  The reading
pinned here: block j's mass is n_tok(j) exp(z_j) with z_j the mean logit
between the q-block's rows and the block's keys, estimated from the pooled
int8 score; k is the shortest prefix of the HRM-first visit order whose
share of the row's mass reaches p.

Every expected value below comes from the mathematics (exact rationals,
closed forms, a construction whose quantisation is exact), not from the
oracle's own arithmetic.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import kap
from synth import from_arrays, make_workload


def _brute_k(z, ntok, p):
    """Smallest prefix whose share >= p, in exact rational arithmetic over the
    fp64 values of n_tok exp(z - max z) (math.exp, one value per block)."""
    zmax = max(z)
    w = [Fraction(int(n)) * Fraction(math.exp(v - zmax)) for v, n in zip(z, ntok)]
    total = sum(w)
    acc = Fraction(0)
    for k, x in enumerate(w, 1):
        acc += x
        if acc / total >= Fraction(p):
            return k, [float(sum(w[:m]) / total) for m in range(1, len(w) + 1)]
    return len(w), None


def test_top_p_brute_force_tiny_rows():
    rng = np.random.default_rng(2024)
    checked = 0
    while checked < 400:
        n = int(rng.integers(1, 13))
        scores = (rng.standard_normal(n) * 3).astype(np.float32)
        ntok = rng.integers(1, 129, n)
        zscale = float(rng.uniform(0.2, 2.0))
        p = float(rng.uniform(0.05, 0.999))
        z = [float(np.float64(s) * zscale) for s in scores]
        want, shares = _brute_k(z, ntok, p)
        if shares is not None and min(abs(x - p) for x in shares) < 1e-9:
            continue                         # too close to a boundary for fp64 to be exact
        k, lo, hi = kap.top_p_count(scores, ntok, zscale, p)
        assert k == want
        assert lo == k == hi                 # far from every boundary: no ambiguity window
        checked += 1


@pytest.mark.parametrize("n", [1, 2, 7, 64, 1000])
def test_top_p_equal_masses_keep_ceil_pn(n):
    """n equal masses: the share of a k-prefix is k/n, so k = ceil(p n)."""
    scores = np.full(n, 0.75, dtype=np.float32)
    ntok = np.full(n, 128)
    for m in range(n):
        p = (m + 0.5) / n                     # strictly between two shares
        assert kap.top_p_count(scores, ntok, 1.3, p)[0] == m + 1 == math.ceil(p * n)


def test_top_p_geometric_masses_closed_form():
    """Masses 2^-j (j = 0..n-1): the k-prefix share is (1 - 2^-k) / (1 - 2^-n)."""
    n = 20
    zscale = 0.5
    scores = np.array([-j * math.log(2.0) / zscale for j in range(n)], dtype=np.float32)
    ntok = np.full(n, 64)
    for k in range(1, n + 1):
        share_prev = (1 - 2.0 ** -(k - 1)) / (1 - 2.0 ** -n)
        share_k = (1 - 2.0 ** -k) / (1 - 2.0 ** -n)
        p = 0.5 * (share_prev + share_k)
        assert kap.top_p_count(scores, ntok, zscale, p)[0] == k


def test_top_p_weights_token_counts_in_visit_order():
    """Two blocks with equal logits and 128 / 64 tokens: shares 2/3 and 1/3."""
    s = np.zeros(2, dtype=np.float32)
    assert kap.top_p_count(s, np.array([128, 64]), 1.0, 0.6)[0] == 1     # 2/3 >= 0.6
    assert kap.top_p_count(s, np.array([128, 64]), 1.0, 0.7)[0] == 2
    assert kap.top_p_count(s, np.array([64, 128]), 1.0, 0.3)[0] == 1     # 1/3 >= 0.3
    assert kap.top_p_count(s, np.array([64, 128]), 1.0, 0.34)[0] == 2


def test_top_p_limits_monotone_and_window():
    rng = np.random.default_rng(7)
    scores = (rng.standard_normal(50) * 4).astype(np.float32)
    ntok = rng.integers(1, 129, 50)
    ks = [kap.top_p_count(scores, ntok, 1.0, p)[0] for p in np.linspace(0.01, 1.0, 200)]
    assert ks == sorted(ks)                          # non-decreasing in p
    assert ks[-1] == 50                              # p = 1 keeps everything
    assert kap.top_p_count(scores, ntok, 1.0, 1e-12)[0] == 1
    # a far tail whose fp64 mass underflows is still kept at p = 1
    far = np.array([0.0, -1000.0, -2000.0], dtype=np.float32)
    assert kap.top_p_count(far, np.array([1, 1, 1]), 1.0, 1.0) == (3, 3, 3)
    assert kap.top_p_count(far, np.array([1, 1, 1]), 1.0, 0.999)[0] == 1
    # p exactly at a share: the window holds both neighbouring cuts
    s = np.zeros(4, dtype=np.float32)
    k, lo, hi = kap.top_p_count(s, np.full(4, 16), 1.0, 0.5)
    assert k == 2 and lo <= 2 and hi >= 3
    for bad in (0.0, -0.1, 1.5):
        with pytest.raises(ValueError):
            kap.top_p_count(s, np.full(4, 16), 1.0, bad)


def _two_block_construction(d=64):
    """L = 96, b = 64: q-block 1 holds 32 rows q = 0.5 (all dims); key block 0
    is 64 keys k = 0.5, key block 1 is 32 keys (+0.5, -0.5 halves).  Every
    pooled vector quantises exactly (its entries share one magnitude), so the
    mean logits are exact: z_0 = q.k_0 / sqrt(d) = 0.25 d / sqrt(d) = 2 at
    d = 64, z_1 = 0.  Block 0's share = 64 e^2 / (64 e^2 + 32)."""
    L, b = 96, 64
    q = np.full((L, 1, d), 0.5, dtype=np.float32)
    k = np.full((L, 1, d), 0.5, dtype=np.float32)
    k[b:, 0, d // 2:] = -0.5
    v = np.ones((L, 1, d), dtype=np.float32)
    return from_arrays([q], [k], [v], b, 32, shuffle=True, seed=5)


def test_top_p_mean_logit_scale_constructed():
    w = _two_block_construction()
    share0 = 64 * math.exp(2.0) / (64 * math.exp(2.0) + 32)        # 0.93661...
    for p, want in ((share0 - 1e-3, 1), (share0 + 1e-3, 2), (0.5, 1), (1.0, 2)):
        r = kap.kap_proxy_top_p(w.q, w.k_pages, w.page_table, w.seqlens, 1, w.block_size, p)
        assert r["count"][0, 0] == 1                                 # one candidate
        assert r["count"][0, 1] == want
        assert r["order"][0, 1, :want].tolist() == [0, 1][:want]
        assert r["hrm"][0, 1, :want].tolist() == [1, 0][:want]
        assert np.all(r["order"][0, 1, want:] == -1)


@pytest.mark.parametrize("p", [0.5, 0.9, 0.95, 1.0])
def test_top_p_cut_is_a_prefix_of_the_full_order(p):
    w = make_workload(1)
    full = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, 1.0)
    r = kap.kap_proxy_top_p(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, p)
    Hq, NQB = r["count"].shape
    for h in range(Hq):
        for i in range(NQB):
            k = int(r["count"][h, i])
            assert 1 <= k <= int(full["count"][h, i])
            assert r["count_lo"][h, i] <= k <= r["count_hi"][h, i]
            assert r["order"][h, i, :k].tolist() == full["order"][h, i, :k].tolist()
            assert r["hrm"][h, i, :k].tolist() == full["hrm"][h, i, :k].tolist()
            assert r["n_hrm"][h, i] == int(r["hrm"][h, i, :k].sum())
            if p == 1.0:
                assert k == full["count"][h, i]

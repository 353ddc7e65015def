"""The register selection's algorithm (select_fast_kernel in kap_stream.cu), modelled on the CPU.

A row's sort keys are 64-bit: bit 63 = not HRM, bits 31..62 = the score's
order-preserving bits (descending in the score), bits 0..30 = the block index.
Rows of at most 32 candidates, or whose budget keeps all, are sorted whole.
Longer rows take the upper 32 bits of 64 keys at evenly spaced positions, a
threshold T at sample rank r = min(63, ceil(64 k / n) + 1), and keep every key
whose upper 32 bits are <= T; if fewer than k are kept, r rises (r + r // 2 + 2,
three passes at most); more than 256 kept, or fewer than k after the last
pass, sends the row to the exact fallback.  The kept set is a down-set of the
key order, so sorting it and taking k gives the k smallest.  This model pins
that claim on random rows (ties, HRM blocks, short and long rows) and checks
that the fallback stays rare.
"""

import numpy as np
import pytest

CAP = 256


def score_bits(s):
    u = np.float32(s).view(np.uint32)
    if (u & np.uint32(0x7FFFFFFF)) == 0:
        u = np.uint32(0)
    asc = ~u if (u & np.uint32(0x80000000)) else (u | np.uint32(0x80000000))
    return int(np.uint32(~asc))


def keys_of(scores, hrm):
    return [((0 if h else 1) << 63) | (score_bits(s) << 31) | j for j, (s, h) in enumerate(zip(scores, hrm))]


def select(keys, k):
    """(the k keys the algorithm returns, whether the row fell back)."""
    n = len(keys)
    if k == n or n <= 32:
        return sorted(keys)[:k], False
    smp = sorted(keys[(e * n) >> 6] >> 32 for e in range(64))
    r = min(63, (64 * k + n - 1) // n + 1)
    kept = []
    for _ in range(3):
        T = smp[r]
        kept = [x for x in keys if (x >> 32) <= T]
        if len(kept) >= k or r == 63:
            break
        r = min(63, r + r // 2 + 2)
    if len(kept) < k or len(kept) > CAP:
        return sorted(keys)[:k], True
    return sorted(kept)[:k], False


def keep_count(n, bp):
    return max(1, (n * bp + 9999) // 10000)


def random_row(rng, n, kind=None):
    kind = rng.integers(4) if kind is None else kind
    if kind == 0:
        s = rng.standard_normal(n).astype(np.float32)
    elif kind == 1:   # heavy ties: few distinct values
        s = rng.integers(-3, 4, n).astype(np.float32)
    elif kind == 2:   # a local band plus a few spikes, as the planted structure
        s = (rng.standard_normal(n) * 0.5 - np.arange(n)[::-1] * 0.01).astype(np.float32)
        s[rng.integers(0, n, 4)] += 5.0
    else:             # zeros of both signs
        s = np.where(rng.random(n) < 0.5, np.float32(0.0), np.float32(-0.0)).astype(np.float32)
    hrm = np.zeros(n, dtype=bool)
    hrm[rng.integers(0, n, rng.integers(1, 9))] = True
    return s, hrm


@pytest.mark.parametrize("bp", [500, 1000, 2000, 10000])
def test_register_selection_returns_the_k_smallest_keys(bp):
    """Every row, whatever its scores (including all-equal and few-valued rows, which the
    threshold cannot split and which take the exact fallback), gets the k smallest keys."""
    rng = np.random.default_rng(bp)
    for _ in range(300):
        n = int(rng.integers(1, 1025))
        s, hrm = random_row(rng, n)
        keys = keys_of(s, hrm)
        k = keep_count(n, bp)
        got, _ = select(keys, k)
        assert got == sorted(keys)[:k]


@pytest.mark.parametrize("bp", [500, 1000])
def test_fallback_is_rare_on_continuous_scores(bp):
    """At the workloads' budgets and with continuous scores the sampled threshold
    finishes the row itself: the exact fallback is the exception."""
    rng = np.random.default_rng(100 + bp)
    fallbacks = rows = 0
    for _ in range(400):
        n = int(rng.integers(33, 1025))
        s, hrm = random_row(rng, n, kind=int(rng.choice([0, 2])))
        keys = keys_of(s, hrm)
        k = keep_count(n, bp)
        got, fb = select(keys, k)
        assert got == sorted(keys)[:k]
        rows += 1
        fallbacks += fb
    assert fallbacks <= 0.05 * rows, fallbacks


def test_a_threshold_that_ignores_the_hrm_flag_is_caught():
    """The model is sensitive: a threshold on the score bits alone (the flag dropped)
    is not a down-set of the key order, and loses a low-scoring HRM block on some row."""
    rng = np.random.default_rng(7)
    wrong = 0
    for _ in range(300):
        n = int(rng.integers(64, 1025))
        s, hrm = random_row(rng, n, kind=0)
        keys = keys_of(s, hrm)
        k = keep_count(n, 500)
        score_hi = lambda x: (x >> 31) & 0xFFFFFFFF
        smp = sorted(score_hi(keys[(e * n) >> 6]) for e in range(64))
        r = min(63, (64 * k + n - 1) // n + 1)
        kept = [x for x in keys if score_hi(x) <= smp[r]]
        if len(kept) >= k and sorted(kept)[:k] != sorted(keys)[:k]:
            wrong += 1
    assert wrong > 0

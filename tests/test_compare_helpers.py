"""The GPU tests' comparison helpers, checked on the CPU with results made by the
oracle itself (no GPU): the parallel oracle pool returns exactly the oracle's
tiles, and compare_attn accepts a faithful result but rejects a corrupted one,
including in a unit whose skip decision legitimately differs inside the window.
"""

import math

import numpy as np
import pytest
import torch

from oracle import kap, osk
from synth import make_custom
from tests import gpu_util as gu
from oracle.parallel import OraclePool


def _fake_gpu(w, ref):
    """Device-style result tensors (on the CPU) carrying the oracle's own answer."""
    out = torch.from_numpy(np.nan_to_num(ref["out"]).astype(np.float32)).to(torch.bfloat16)
    return dict(out=out, visited=torch.from_numpy(ref["visited"].copy()),
                skipped=torch.from_numpy(ref["skipped"].copy()),
                skipbits=torch.from_numpy(ref["skip"].astype(np.uint8)))


@pytest.fixture(scope="module")
def small():
    w = make_custom([700, 300], 4, 2, 64, 64, 32, structure="llama", seed=11)
    sel = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, 0.3)
    return w, sel


def test_pool_returns_the_oracles_tiles(small):
    w, sel = small
    units = gu.sample_units(w, 40, seed=3)
    full = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size,
                   sel["order"], sel["count"], 1e-3, units=units)
    with OraclePool(w, workers=2) as pool:
        got = pool.run(sel["order"], sel["count"], 1e-3, units)
    assert sorted(got) == sorted(units)
    for (h, I), (rows, o, sk, de) in got.items():
        np.testing.assert_array_equal(o, full["out"][rows, h])
        np.testing.assert_array_equal(sk, full["skip"][h, I, :len(sk)])
        np.testing.assert_array_equal(de, full["delta"][h, I, :len(de)])
        assert len(sk) == full["visited"][h, I]


def _window_case(w, sel):
    """tau placed on one visited block's statistic, so that flipping that block's
    decision is legitimate (|delta - ln tau| = 0 <= window)."""
    probe = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size,
                    sel["order"], sel["count"], 0.0)
    cand = [(probe["delta"][h, I, t], h, I, t) for h in range(w.num_q_heads) for I in range(sel["order"].shape[1])
            for t in range(1, int(sel["count"][h, I])) if np.isfinite(probe["delta"][h, I, t])]
    _, h, I, t = min(cand)            # the most negligible block: the smallest tau, the tightest allowance
    tau = math.exp(probe["delta"][h, I, t])
    ref = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size,
                  sel["order"], sel["count"], tau)
    return tau, ref, (h, I, t)


def test_compare_attn_accepts_the_oracle_and_a_window_flip(small):
    w, sel = small
    tau, ref, (h, I, t) = _window_case(w, sel)
    res = _fake_gpu(w, ref)
    gu.compare_attn(res, ref, w, tau, gu.all_units(w))
    # the kernel may decide the other way on a block inside the window
    flip = 1 - int(res["skipbits"][h, I, t])
    res["skipbits"][h, I, t] = flip
    res["skipped"][h, I] += 1 if flip else -1
    stats = gu.compare_attn(res, ref, w, tau, gu.all_units(w))
    assert stats["exempt_units"] == 1 and stats["flipped_blocks"] == 1


def test_compare_attn_rejects_a_wrong_exempt_unit(small):
    w, sel = small
    tau, ref, (h, I, t) = _window_case(w, sel)
    res = _fake_gpu(w, ref)
    flip = 1 - int(res["skipbits"][h, I, t])
    res["skipbits"][h, I, t] = flip
    res["skipped"][h, I] += 1 if flip else -1
    b = w.block_size
    L0 = w.seqlens[0]
    row = I * b if I * b < L0 else L0 + (I - (L0 + b - 1) // b) * b
    allow = gu.MAX_ABS + 2.0 * b * tau * math.exp(gu.DELTA_WINDOW) * gu._max_abs_v(w)
    res["out"][row, h, 0] += 4.0 * allow + 0.1      # far beyond the flipped block's allowance
    with pytest.raises(AssertionError, match="flipped blocks"):
        gu.compare_attn(res, ref, w, tau, gu.all_units(w))


def test_compare_attn_rejects_a_skip_count_that_disagrees_with_the_bits(small):
    w, sel = small
    ref = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size,
                  sel["order"], sel["count"], 1e-3)
    res = _fake_gpu(w, ref)
    res["skipped"][0, 3] += 1
    with pytest.raises(AssertionError, match="skip bits"):
        gu.compare_attn(res, ref, w, 1e-3, gu.all_units(w))

"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (same entry points, same shapes).

* Proxy: every (head, q-block) row bit-exact against the oracle.
* Attention: a seeded sample of (head, q-block) tiles per budget and tau,
  always including each sequence's first and last q-block (ragged tails),
  compared element by element (the oracle computes tiles independently).
"""

import gc

import numpy as np
import pytest
import torch

import block_sparse_long_14_b200 as cosa
from oracle import kap, osk
from synth import make_workload
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

SAMPLE_TILES = 40


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_full_size_workload(cfg):
    w = make_workload(cfg)
    d = gu.upload(w)
    try:
        for budget in w.budgets:
            got, kmax, ws = gu.run_proxy(d, budget)
            ref = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, budget)
            assert kmax == ref["kmax"]
            gu.assert_proxy_equal(got, ref)
            sel = dict(order=torch.from_numpy(got["order"]).cuda(), count=torch.from_numpy(got["count"]).cuda())
            units = gu.all_units(w) if cfg == 1 else gu.sample_units(w, SAMPLE_TILES, seed=cfg)
            for tau in w.taus:
                res = gu.run_attn(d, sel, kmax, tau, ws)
                o = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size,
                            ref["order"], ref["count"], tau, units=units)
                stats = gu.compare_attn(res, o, w, tau, units)
                print(f"cfg {cfg} budget {budget} tau {tau}: {stats}")
                del res
            del sel, ws
    finally:
        del d
        gc.collect()
        torch.cuda.empty_cache()

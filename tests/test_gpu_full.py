"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (same entry points, same shapes).

* Proxy: every (head, q-block) row bit-exact against the oracle.
* Attention: every (head, q-block) tile at the 32K and 64K layers (and the
  tiny one); at the 128K layer and the ragged batch a seeded 10 % of the
  tiles, always including each sequence's first and last q-block for every
  head (the ragged tails), compared element by element for every budget and
  tau.  The oracle computes tiles independently, so they are evaluated in
  parallel CPU processes (oracle/parallel.py).
"""

import gc
import math

import numpy as np
import pytest
import torch

from oracle import kap
from synth import make_workload
from tests import gpu_util as gu
from oracle.parallel import OraclePool

pytestmark = pytest.mark.gpu

EVERY_TILE = {1, 2, 4}
SAMPLE_FRACTION = 0.10


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_full_size_workload(cfg):
    w = make_workload(cfg)
    d = gu.upload(w)
    total = w.num_q_heads * d["batch"].total_qblocks
    units = gu.all_units(w) if cfg in EVERY_TILE else gu.sample_units(w, math.ceil(SAMPLE_FRACTION * total), seed=cfg)
    try:
        with OraclePool(w) as pool:
            for budget in w.budgets:
                got, kmax, ws = gu.run_proxy(d, budget)
                ref = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, budget)
                assert kmax == ref["kmax"]
                gu.assert_proxy_equal(got, ref)
                sel = dict(order=torch.from_numpy(got["order"]).cuda(), count=torch.from_numpy(got["count"]).cuda())
                for tau in w.taus:
                    res = gu.run_attn(d, sel, kmax, tau, ws)
                    o = pool.run(ref["order"], ref["count"], tau, units)
                    stats = gu.compare_attn(res, o, w, tau, units)
                    print(f"cfg {cfg} budget {budget} tau {tau}: {stats}")
                    assert stats["units"] == len(units)
                    del res, o
                del sel, ws
    finally:
        del d
        gc.collect()
        torch.cuda.empty_cache()

"""Failure detection through the C ABI, without faulting the GPU.

* Argument errors are caught on the host before anything is enqueued.
* A pipeline wait cap far too small for the pipeline makes the attention
  kernel, and the persistent proxy kernel, record COSA_ERR_TIMEOUT, drain
  their own copies and MMAs, free TMEM and return; the context stays usable
  and the next call is correct.
* A block index outside the sequence is caught by the kernels' bounds checks
  (reported as COSA_ERR_DEVICE; the access is skipped).
"""

import numpy as np
import pytest
import torch

import block_sparse_long_14_b200 as cosa
from oracle import kap, osk
from synth import make_custom
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _case():
    w = make_custom([700, 300], 8, 2, 128, 128, 64, structure="llama", seed=31)
    return w, gu.upload(w)


def test_argument_errors_are_reported_on_the_host():
    w, d = _case()
    ws, kmax = cosa.alloc_workspace(d["batch"], 0.25)
    sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], 0.25, kmax, ws)
    with pytest.raises(cosa.CosaError) as e:
        cosa.attn(d["batch"], d["q"], d["k_pages"], d["v_pages"], d["page_table"], sel["order"], sel["count"],
                  kmax, 1.0, ws)
    assert e.value.code == 1
    with pytest.raises(cosa.CosaError) as e:
        cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], 0.0, kmax, ws)
    assert e.value.code == 1
    with pytest.raises(cosa.CosaError) as e:
        cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], 0.25, kmax, ws[:64])
    assert e.value.code == 3
    with pytest.raises(cosa.CosaError) as e:   # kmax too small for the budget
        cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], 0.25, 1, ws)
    assert e.value.code == 1
    cosa.check(ws)


def test_injected_wait_timeout_is_reported_and_recoverable():
    w, d = _case()
    ws, kmax = cosa.alloc_workspace(d["batch"], 0.25)
    sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], 0.25, kmax, ws)
    cosa.check(ws)
    try:
        cosa.set_wait_limit(1)
        cosa.attn(d["batch"], d["q"], d["k_pages"], d["v_pages"], d["page_table"], sel["order"], sel["count"],
                  kmax, 1e-4, ws)
        with pytest.raises(cosa.CosaError) as e:
            cosa.check(ws)
        assert e.value.code == 5
    finally:
        cosa.set_wait_limit(0)
    # the context is intact and the status word was cleared
    res = gu.run_attn(d, sel, kmax, 1e-4, ws)
    ref_sel = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, 2, 128, 0.25)
    ref = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, 2, 128, ref_sel["order"],
                  ref_sel["count"], 1e-4)
    gu.compare_attn(res, ref, w, 1e-4, gu.all_units(w))


def test_injected_wait_timeout_in_the_proxy_is_reported_and_recoverable():
    """The same for the persistent proxy kernel (head_dim 128, budget cut): every role's
    wait gives up, the CTA drains its copies and MMAs and frees TMEM, the selection kernels
    run on whatever was written (in bounds), the status reports the timeout, and the next
    call is bit-exact."""
    w, d = _case()
    ws, kmax = cosa.alloc_workspace(d["batch"], 0.25)
    try:
        cosa.set_wait_limit(1)
        cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], 0.25, kmax, ws)
        with pytest.raises(cosa.CosaError) as e:
            cosa.check(ws)
        assert e.value.code == 5
    finally:
        cosa.set_wait_limit(0)
    got, kmax2, _ = gu.run_proxy(d, 0.25)
    ref = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, 2, 128, 0.25)
    assert kmax2 == ref["kmax"]
    gu.assert_proxy_equal(got, ref)


def test_out_of_range_block_is_caught_by_bounds_checks():
    w, d = _case()
    ws, kmax = cosa.alloc_workspace(d["batch"], 0.25)
    sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], 0.25, kmax, ws)
    cosa.check(ws)
    bad = sel["order"].clone()
    bad[0, 3, 0] = 10_000
    cosa.attn(d["batch"], d["q"], d["k_pages"], d["v_pages"], d["page_table"], bad, sel["count"], kmax, 1e-4, ws)
    with pytest.raises(cosa.CosaError) as e:
        cosa.check(ws)
    assert e.value.code == 6
    cosa.remap(d["batch"], d["page_table"], bad, sel["count"], kmax)
    torch.cuda.synchronize()
    cosa.check(ws)   # remap reports nothing into the workspace; the bad entry maps to -1

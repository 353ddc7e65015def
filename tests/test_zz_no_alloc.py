"""cosa_proxy_noalloc: the proxy for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: code running inside an inference engine
that has reserved nearly all device memory for its own pools and offers no
scratch API, or code on a latency-critical path.  For them the library keeps
the proxy's pooled-key scratch in a fixed static device array.  This file
checks, through the C ABI, that this entry point returns exactly what the
workspace-based cosa_proxy returns (block lists are integer results: the
tolerance is bit-exactness), on two calls in a row with different inputs so
that the array's leftover contents from the first call cannot leak into the
second, and that a shape needing more scratch than the array holds is refused
before anything is enqueued.

It lives in a file of its own, collected last, and needs nothing from the
other test files.
"""

import numpy as np
import pytest
import torch

import block_sparse_long_14_b200 as cosa
from synth import make_custom

pytestmark = pytest.mark.gpu


def _upload(w):
    def bf16(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()

    batch = cosa.Batch(w.seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.page_size,
                       w.num_pages, w.max_pages_per_seq)
    return batch, bf16(w.q), bf16(w.k_pages), torch.from_numpy(np.ascontiguousarray(w.page_table)).cuda()


def test_noalloc_proxy_matches_workspace_proxy_on_two_calls_in_a_row():
    cases = [
        (make_custom([3000, 700, 129], 8, 2, 128, 128, 64, structure="llama", seed=41), 0.10),
        (make_custom([1500, 64], 16, 4, 64, 64, 32, structure="llama", seed=42), 0.25),
    ]
    for w, budget in cases:
        batch, q, kp, pt = _upload(w)
        ws, kmax = cosa.alloc_workspace(batch, budget)
        ref = cosa.proxy(batch, q, kp, pt, budget, kmax, ws)
        cosa.check(ws)
        got = cosa.proxy_noalloc(batch, q, kp, pt, budget, kmax)
        torch.cuda.synchronize()
        for key in ("order", "count", "n_hrm", "hrm"):
            assert torch.equal(got[key], ref[key]), key


def test_noalloc_proxy_refuses_shapes_beyond_its_scratch():
    # 8 kv heads x 4096 q-blocks: 4 MiB of int8 keys + 128 KiB of scales > 4 MiB,
    # refused on the host before anything is read
    L = 4096 * 128
    batch = cosa.Batch([L], 32, 8, 128, 128, 64, num_pages=L // 64, max_pages_per_seq=L // 64)
    _, kmax = cosa.workspace_size(batch, 0.05)
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    table = torch.zeros(16, dtype=torch.int32, device="cuda")
    out = dict(order=torch.empty(16, dtype=torch.int32, device="cuda"),
               count=torch.empty(16, dtype=torch.int32, device="cuda"),
               n_hrm=torch.empty(16, dtype=torch.int32, device="cuda"),
               hrm=torch.empty(16, dtype=torch.uint8, device="cuda"))
    with pytest.raises(cosa.CosaError) as e:
        cosa.proxy_noalloc(batch, dummy, dummy, table, 0.05, kmax, out=out)
    assert e.value.code == 3

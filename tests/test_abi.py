"""The C ABI library on the host (no GPU needed): it builds for sm_100a, loads,
exports every entry point include/cosa.h declares, and its host-side logic
(argument checks, workspace sizing, list length kmax) behaves as declared.
No call here launches a kernel.
"""

import ctypes
import os
import re
import subprocess

import pytest

import block_sparse_long_14_b200 as cosa
from block_sparse_long_14_b200 import build as cbuild
from oracle import kap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cosa.h")


@pytest.fixture(scope="module")
def lib():
    cbuild.build()
    return cosa.lib()


def declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"COSA_API\s+[\w\s\*]+?\b(cosa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared()
    for n in ("cosa_proxy", "cosa_remap", "cosa_attn", "cosa_workspace_size", "cosa_sync_status"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", cosa.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (cosa_\w+)", out))
    assert set(declared()) <= exported
    for n in declared():
        assert hasattr(lib, n)


def test_library_is_built_for_sm100a(lib):
    out = subprocess.run(["cuobjdump", "--list-elf", cosa.LIB_PATH], capture_output=True, text=True)
    if out.returncode == 0:
        assert "sm_100a" in out.stdout


def test_error_strings(lib):
    for code in range(7):
        assert lib.cosa_error_string(code)
    assert lib.cosa_version() >= 100


def _shape(**kw):
    base = dict(batch=1, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=128, page_size=64,
                num_pages=2048, max_pages_per_seq=2048, total_tokens=131072, total_qblocks=1024,
                max_seqlen=131072, cu_seqlens=16, cu_qblocks=32)   # pointers are not dereferenced here
    base.update(kw)
    return cosa._Shape(**base)


def _ws(shape, budget):
    k = ctypes.c_int32(0)
    n = cosa.lib().cosa_workspace_size(ctypes.byref(shape), ctypes.c_float(budget), ctypes.byref(k))
    return n, k.value


@pytest.mark.parametrize("budget", [0.05, 0.1, 0.2, 0.25, 1.0])
@pytest.mark.parametrize("max_seqlen,b", [(131072, 128), (90000, 128), (1024, 64), (1, 128)])
def test_workspace_size_and_kmax(lib, budget, max_seqlen, b):
    nqb = (max_seqlen + b - 1) // b
    sh = _shape(block_size=b, max_seqlen=max_seqlen, total_tokens=max_seqlen, total_qblocks=nqb,
                max_pages_per_seq=(max_seqlen + 63) // 64)
    n, kmax = _ws(sh, budget)
    assert kmax == kap.kmax_for(nqb, budget)
    assert n >= 256 + 8 * nqb * 128 + 8 * nqb * 4 and n % 256 == 0


@pytest.mark.parametrize("bad", [
    dict(head_dim=96), dict(block_size=256), dict(page_size=48), dict(page_size=4), dict(num_kv_heads=5),
    dict(num_q_heads=64, num_kv_heads=4), dict(max_pages_per_seq=10), dict(cu_seqlens=0), dict(batch=0),
    dict(total_qblocks=3),
])
def test_invalid_shapes_are_rejected(lib, bad):
    assert _ws(_shape(**bad), 0.1)[0] == 0


def test_invalid_budgets_are_rejected(lib):
    for b in (0.0, -0.1, 1.5, float("nan")):
        assert _ws(_shape(), b)[0] == 0


def test_null_pointers_rejected_before_launch(lib):
    sh = _shape()
    rc = lib.cosa_proxy(ctypes.byref(sh), None, None, None, ctypes.c_float(0.1), 64, None, None, None, None, None,
                        0, None)
    assert rc == 1
    rc = lib.cosa_attn(ctypes.byref(sh), None, None, None, None, None, None, 52, ctypes.c_float(1e-4), None, None,
                       None, None, None, 0, None)
    assert rc == 1
    rc = lib.cosa_remap(ctypes.byref(sh), None, None, None, 52, None, None)
    assert rc == 1


@pytest.mark.parametrize("delta", [0.0, -0.5, -2.0, float("nan"), float("inf")])
def test_attn_delta_rejects_bad_delta(lib, delta):
    sh = _shape()
    rc = lib.cosa_attn_delta(ctypes.byref(sh), None, None, None, None, None, None, 52, ctypes.c_float(delta), None,
                             None, None, None, None, 0, None)
    assert rc == 1


def test_attn_rejects_tau_outside_unit_interval(lib):
    sh = _shape()
    for tau in (-1e-3, 1.0, 2.0, float("nan")):
        rc = lib.cosa_attn(ctypes.byref(sh), None, None, None, None, None, None, 52, ctypes.c_float(tau), None,
                           None, None, None, None, 0, None)
        assert rc == 1


def test_attn_masked_needs_a_keep_mask(lib):
    sh = _shape()
    rc = lib.cosa_attn_masked(ctypes.byref(sh), None, None, None, None, None, None, 1024, None, ctypes.c_float(1e-4),
                              None, None, None, None, None, 0, None)
    assert rc == 1


def test_page_layouts(lib):
    assert _ws(_shape(page_layout=0), 0.1)[0] > 0
    assert _ws(_shape(page_layout=1), 0.1)[0] > 0
    assert _ws(_shape(page_layout=2), 0.1)[0] == 0
    assert lib.cosa_version() >= 101


def test_cached_prefix_shape_checks(lib):
    """kv_lens set: the key blocks are counted apart from the q-blocks, the
    workspace's pooled keys follow NKB, and inconsistent counts are refused."""
    # 128K keys, the last 8K tokens are queries: 64 present q-blocks of 1024 key blocks
    ok = dict(total_tokens=8192, total_qblocks=64, max_seqlen=131072, kv_lens=48, cu_kblocks=64,
              total_kblocks=1024)
    n_prefix, kmax = _ws(_shape(**ok), 0.05)
    assert kmax == kap.kmax_for(1024, 0.05)          # lists sized by the longest key sequence
    n_full, _ = _ws(_shape(), 0.05)
    # pooled keys and scales sized by NKB (same as full prefill); query vectors and their
    # scales, each row's candidate score bits (the longest sequence's 1024 key blocks), its 8
    # HRM slots and its retry-list entry by NQB only
    per_qblock = 32 * 9 * 128 + 32 * 4 + 32 * 1024 * 4 + 32 * 8 * 4 + 32 * 4
    assert n_full - n_prefix == (1024 - 64) * per_qblock
    for bad in (dict(cu_kblocks=0), dict(total_kblocks=0), dict(total_kblocks=1023), dict(total_kblocks=63,
                max_seqlen=8000)):
        assert _ws(_shape(**{**ok, **bad}), 0.05)[0] == 0, bad
    # without kv_lens the old rule holds: every token a query, max_seqlen <= total_tokens
    assert _ws(_shape(total_tokens=8192, total_qblocks=64, max_seqlen=131072), 0.05)[0] == 0
    assert lib.cosa_version() >= 102


def test_batch_prefix_offsets_on_the_host():
    """Batch's offset arrays for a cached prefix, checked on the CPU."""
    b = cosa.Batch([300, 128, 133], 4, 2, 64, 64, 16, 64, 8, device="cpu", q_lens=[100, 128, 1])
    assert b.cu_seqlens.tolist() == [0, 100, 228, 229]
    # q-blocks holding a query row: 5 - 200//64, 2 - 0, 3 - 132//64
    assert b.cu_qblocks.tolist() == [0, 2, 4, 5]
    assert b.cu_kblocks.tolist() == [0, 5, 7, 10]
    assert b.kv_lens.tolist() == [300, 128, 133]
    assert (b.total_tokens, b.total_qblocks, b.total_kblocks) == (229, 5, 10)
    assert b.c.total_kblocks == 10 and b.c.max_seqlen == 300
    full = cosa.Batch([300, 128], 4, 2, 64, 64, 16, 64, 8, device="cpu")
    assert full.kv_lens is None and full.c.kv_lens is None and full.c.total_kblocks == 0
    for bad in ([0, 128, 1], [301, 128, 1], [1, 1]):
        with pytest.raises(ValueError):
            cosa.Batch([300, 128, 133], 4, 2, 64, 64, 16, 64, 8, device="cpu", q_lens=bad)


def test_proxy_top_p_arguments(lib):
    """cosa_proxy_top_p: p in (0, 1]; kmax must cover every candidate."""
    sh = _shape()
    n_all = 1024

    def call(p, kmax):
        return lib.cosa_proxy_top_p(ctypes.byref(sh), 16, 16, 16, ctypes.c_float(p), kmax, 16, 16, 16, 16, 256,
                                    1 << 40, None)
    for p in (0.0, -0.5, 1.5, float("nan")):
        assert call(p, n_all) == 1
    assert call(0.95, n_all - 1) == 1        # a row may keep all of its candidates
    rc = lib.cosa_proxy_top_p(ctypes.byref(sh), None, None, None, ctypes.c_float(0.95), n_all, None, None, None,
                              None, None, 0, None)
    assert rc == 1
    assert _ws(sh, 1.0)[1] == n_all         # budget 1.0 reports the kmax Top-p needs


def test_noalloc_scratch_boundary(lib):
    """cosa_proxy_noalloc keeps the pooled keys (Hkv x NKB x d int8, rounded up to
    256 bytes) and their scales (Hkv x NKB fp32) in its fixed array: 8 kv heads
    at d = 128 take 1,056 bytes per key block, so 3,971 key blocks fit in
    COSA_NOALLOC_SCRATCH_BYTES and 3,972 are refused with COSA_ERR_WORKSPACE
    before anything reaches the device."""
    import torch
    limit = 4 << 20

    def need(nkb):
        return (8 * nkb * 128 + 255) // 256 * 256 + 8 * nkb * 4

    assert need(3971) <= limit < need(3972)
    fake = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced on the refusing path

    def call(nkb):
        L = nkb * 128
        sh = _shape(total_tokens=L, total_qblocks=nkb, max_seqlen=L, num_pages=nkb * 2, max_pages_per_seq=nkb * 2)
        return lib.cosa_proxy_noalloc(ctypes.byref(sh), fake, fake, fake, ctypes.c_float(0.05), 256, fake, fake,
                                      fake, fake, None)

    assert call(3972) == 3
    if not torch.cuda.is_available():
        # without a device the accepted size fails later, at the device query, never at the size check
        assert call(3971) not in (0, 3)

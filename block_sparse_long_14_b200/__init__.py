"""CoSA prefill path on B200: Python binding of libcosa (include/cosa.h).

Argument marshalling only.  Every step of the path runs in libcosa's CUDA
kernels; PyTorch supplies device memory and the current stream.  There is
no CPU or PyTorch fallback: if the library is missing or a call fails, an
exception is raised.

    batch = Batch(seqlens, Hq, Hkv, d, b, b_p, num_pages, max_pages, device)
    ws, kmax = alloc_workspace(batch, budget)
    sel = proxy(batch, q, k_pages, page_table, budget, kmax, ws)
    res = attn(batch, q, k_pages, v_pages, page_table, sel["order"], sel["count"], kmax, tau, ws)
    check(ws)     # synchronises; raises CosaError on a device-side error
"""

from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "Batch", "CosaError", "PAGES_HND", "PAGES_NHD", "alloc_workspace", "attn", "attn_delta", "attn_masked", "check", "lib", "proxy", "proxy_top_p", "remap",
    "set_wait_limit", "workspace_size", "LIB_PATH",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcosa.so")

COSA_OK = 0
STATUS_NAMES = {0: "COSA_OK", 1: "COSA_ERR_INVALID_ARG", 2: "COSA_ERR_UNSUPPORTED", 3: "COSA_ERR_WORKSPACE",
                4: "COSA_ERR_CUDA", 5: "COSA_ERR_TIMEOUT", 6: "COSA_ERR_DEVICE"}


class CosaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)} ({_lib().cosa_error_string(code).decode()})")


class _Shape(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32), ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32), ("total_tokens", ctypes.c_int32),
        ("total_qblocks", ctypes.c_int32), ("max_seqlen", ctypes.c_int32),
        ("cu_seqlens", ctypes.c_void_p), ("cu_qblocks", ctypes.c_void_p), ("page_layout", ctypes.c_int32),
        ("kv_lens", ctypes.c_void_p), ("cu_kblocks", ctypes.c_void_p), ("total_kblocks", ctypes.c_int32),
    ]


PAGES_HND = 0   # k/v pages [P, Hkv, b_p, d]
PAGES_NHD = 1   # k/v pages [P, b_p, Hkv, d]


_P = ctypes.c_void_p
_SIGS = {
    "cosa_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(_Shape), ctypes.c_float, ctypes.POINTER(ctypes.c_int32)]),
    "cosa_workspace_init": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "cosa_proxy": (ctypes.c_int, [ctypes.POINTER(_Shape), _P, _P, _P, ctypes.c_float, ctypes.c_int32,
                                  _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "cosa_proxy_noalloc": (ctypes.c_int, [ctypes.POINTER(_Shape), _P, _P, _P, ctypes.c_float, ctypes.c_int32,
                                          _P, _P, _P, _P, _P]),
    "cosa_proxy_top_p": (ctypes.c_int, [ctypes.POINTER(_Shape), _P, _P, _P, ctypes.c_float, ctypes.c_int32,
                                        _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "cosa_remap": (ctypes.c_int, [ctypes.POINTER(_Shape), _P, _P, _P, ctypes.c_int32, _P, _P]),
    "cosa_attn": (ctypes.c_int, [ctypes.POINTER(_Shape), _P, _P, _P, _P, _P, _P, ctypes.c_int32, ctypes.c_float,
                                 _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "cosa_attn_delta": (ctypes.c_int, [ctypes.POINTER(_Shape), _P, _P, _P, _P, _P, _P, ctypes.c_int32,
                                       ctypes.c_float, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "cosa_attn_masked": (ctypes.c_int, [ctypes.POINTER(_Shape), _P, _P, _P, _P, _P, _P, ctypes.c_int32, _P,
                                        ctypes.c_float, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "cosa_sync_status": (ctypes.c_int, [_P, _P]),
    "cosa_debug_set_wait_limit": (None, [ctypes.c_uint32]),
    "cosa_error_string": (ctypes.c_char_p, [ctypes.c_int]),
    "cosa_version": (ctypes.c_int, []),
}

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run `python -m block_sparse_long_14_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def lib():
    """The loaded libcosa (ctypes.CDLL)."""
    return _lib()


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t, dtype, what):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{what}: expected a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{what}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what}: must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _check(rc, what):
    if rc != COSA_OK:
        raise CosaError(rc, what)


class Batch:
    """Shape of one packed prefill batch; owns the device offset arrays.

    seqlens: tokens per sequence (keys).  q_lens: optional queries per
    sequence for prefill after a cached prefix; query t of sequence s is
    token seqlens[s] - q_lens[s] + t, and q/out hold only the query rows.
    Default: every token is a query.
    """

    def __init__(self, seqlens, num_q_heads, num_kv_heads, head_dim, block_size, page_size, num_pages,
                 max_pages_per_seq, device="cuda", page_layout=PAGES_HND, q_lens=None):
        self.seqlens = [int(x) for x in seqlens]
        self.q_lens = list(self.seqlens) if q_lens is None else [int(x) for x in q_lens]
        if len(self.q_lens) != len(self.seqlens):
            raise ValueError("q_lens and seqlens differ in length")
        if any(not 1 <= Lq <= L for L, Lq in zip(self.seqlens, self.q_lens)):
            raise ValueError("need 1 <= q_len <= seqlen for every sequence")
        b = int(block_size)
        cu_s, cu_q, cu_k = [0], [0], [0]
        for L, Lq in zip(self.seqlens, self.q_lens):
            nkb = (L + b - 1) // b
            cu_s.append(cu_s[-1] + Lq)
            cu_q.append(cu_q[-1] + nkb - (L - Lq) // b)    # q-blocks that hold a query row
            cu_k.append(cu_k[-1] + nkb)
        self.cu_seqlens = torch.tensor(cu_s, dtype=torch.int32, device=device)
        self.cu_qblocks = torch.tensor(cu_q, dtype=torch.int32, device=device)
        self.prefix = q_lens is not None
        self.kv_lens = torch.tensor(self.seqlens, dtype=torch.int32, device=device) if self.prefix else None
        self.cu_kblocks = torch.tensor(cu_k, dtype=torch.int32, device=device) if self.prefix else None
        self.num_q_heads, self.num_kv_heads, self.head_dim = int(num_q_heads), int(num_kv_heads), int(head_dim)
        self.block_size, self.page_size = b, int(page_size)
        self.total_tokens, self.total_qblocks, self.total_kblocks = cu_s[-1], cu_q[-1], cu_k[-1]
        self.c = _Shape(len(self.seqlens), self.num_q_heads, self.num_kv_heads, self.head_dim, b, self.page_size,
                        int(num_pages), int(max_pages_per_seq), self.total_tokens, self.total_qblocks,
                        max(self.seqlens), self.cu_seqlens.data_ptr(), self.cu_qblocks.data_ptr(),
                        int(page_layout),
                        self.kv_lens.data_ptr() if self.prefix else None,
                        self.cu_kblocks.data_ptr() if self.prefix else None,
                        self.total_kblocks if self.prefix else 0)


def workspace_size(batch: Batch, budget: float):
    """(bytes, kmax) for this batch and stage-1 budget."""
    kmax = ctypes.c_int32(0)
    n = _lib().cosa_workspace_size(ctypes.byref(batch.c), ctypes.c_float(budget), ctypes.byref(kmax))
    if n == 0:
        raise CosaError(1, "cosa_workspace_size")
    return int(n), int(kmax.value)


def alloc_workspace(batch: Batch, budget: float):
    """A zeroed workspace tensor (uint8, 256-byte aligned by the caching allocator) and kmax."""
    n, kmax = workspace_size(batch, budget)
    ws = torch.zeros(n, dtype=torch.uint8, device=batch.cu_seqlens.device)
    return ws, kmax


def proxy(batch: Batch, q, k_pages, page_table, budget: float, kmax: int, workspace, out=None):
    """KAP: ordered block lists.  Returns dict(order, count, n_hrm, hrm)."""
    H, N = batch.num_q_heads, batch.total_qblocks
    dev = q.device
    if out is None:
        out = dict(order=torch.empty((H, N, kmax), dtype=torch.int32, device=dev),
                   count=torch.empty((H, N), dtype=torch.int32, device=dev),
                   n_hrm=torch.empty((H, N), dtype=torch.int32, device=dev),
                   hrm=torch.empty((H, N, kmax), dtype=torch.uint8, device=dev))
    rc = _lib().cosa_proxy(ctypes.byref(batch.c), _ptr(q, torch.bfloat16, "q"), _ptr(k_pages, torch.bfloat16, "k_pages"),
                           _ptr(page_table, torch.int32, "page_table"), ctypes.c_float(budget), int(kmax),
                           _ptr(out["order"], torch.int32, "order"), _ptr(out["count"], torch.int32, "count"),
                           _ptr(out["n_hrm"], torch.int32, "n_hrm"), _ptr(out["hrm"], torch.uint8, "hrm"),
                           _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream())
    _check(rc, "cosa_proxy")
    return out


def proxy_top_p(batch: Batch, q, k_pages, page_table, p: float, kmax: int, workspace, out=None):
    """KAP with the Top-p stage-1 cut (cosa_proxy_top_p).  kmax must cover
    every candidate: alloc_workspace(batch, 1.0) returns it."""
    H, N = batch.num_q_heads, batch.total_qblocks
    dev = q.device
    if out is None:
        out = dict(order=torch.empty((H, N, kmax), dtype=torch.int32, device=dev),
                   count=torch.empty((H, N), dtype=torch.int32, device=dev),
                   n_hrm=torch.empty((H, N), dtype=torch.int32, device=dev),
                   hrm=torch.empty((H, N, kmax), dtype=torch.uint8, device=dev))
    rc = _lib().cosa_proxy_top_p(ctypes.byref(batch.c), _ptr(q, torch.bfloat16, "q"),
                                 _ptr(k_pages, torch.bfloat16, "k_pages"), _ptr(page_table, torch.int32, "page_table"),
                                 ctypes.c_float(p), int(kmax), _ptr(out["order"], torch.int32, "order"),
                                 _ptr(out["count"], torch.int32, "count"), _ptr(out["n_hrm"], torch.int32, "n_hrm"),
                                 _ptr(out["hrm"], torch.uint8, "hrm"), _ptr(workspace, torch.uint8, "workspace"),
                                 workspace.numel(), _stream())
    _check(rc, "cosa_proxy_top_p")
    return out


def proxy_noalloc(batch: Batch, q, k_pages, page_table, budget: float, kmax: int, out=None):
    """KAP without a workspace, for callers that cannot allocate device memory.

    The pooled keys go to the library's fixed static device scratch array
    instead (see cosa_proxy_noalloc in include/cosa.h for its size limit and
    its sharing rules).  The output lists are still the caller's: pass them
    in `out` to avoid any allocation here.
    """
    H, N = batch.num_q_heads, batch.total_qblocks
    dev = q.device
    if out is None:
        out = dict(order=torch.empty((H, N, kmax), dtype=torch.int32, device=dev),
                   count=torch.empty((H, N), dtype=torch.int32, device=dev),
                   n_hrm=torch.empty((H, N), dtype=torch.int32, device=dev),
                   hrm=torch.empty((H, N, kmax), dtype=torch.uint8, device=dev))
    rc = _lib().cosa_proxy_noalloc(ctypes.byref(batch.c), _ptr(q, torch.bfloat16, "q"),
                                   _ptr(k_pages, torch.bfloat16, "k_pages"), _ptr(page_table, torch.int32, "page_table"),
                                   ctypes.c_float(budget), int(kmax), _ptr(out["order"], torch.int32, "order"),
                                   _ptr(out["count"], torch.int32, "count"), _ptr(out["n_hrm"], torch.int32, "n_hrm"),
                                   _ptr(out["hrm"], torch.uint8, "hrm"), _stream())
    _check(rc, "cosa_proxy_noalloc")
    return out


def remap(batch: Batch, page_table, order, count, kmax: int, pages=None):
    """Ordered block lists -> physical page lists [Hq, NQB, kmax * b / b_p]."""
    ppb = batch.block_size // batch.page_size
    if pages is None:
        pages = torch.empty((batch.num_q_heads, batch.total_qblocks, kmax * ppb), dtype=torch.int32,
                            device=order.device)
    rc = _lib().cosa_remap(ctypes.byref(batch.c), _ptr(page_table, torch.int32, "page_table"),
                           _ptr(order, torch.int32, "order"), _ptr(count, torch.int32, "count"), int(kmax),
                           _ptr(pages, torch.int32, "pages"), _stream())
    _check(rc, "cosa_remap")
    return pages


def _attn(entry, batch: Batch, q, k_pages, v_pages, page_table, order, count, kmax: int, thr: float, workspace,
          out, skipbits: bool, keep=None):
    H, N = batch.num_q_heads, batch.total_qblocks
    dev = q.device
    res = out if out is not None else dict(
        out=torch.empty_like(q),
        visited=torch.empty((H, N), dtype=torch.int32, device=dev),
        skipped=torch.empty((H, N), dtype=torch.int32, device=dev))
    if skipbits and "skipbits" not in res:
        res["skipbits"] = torch.empty((H, N, kmax), dtype=torch.uint8, device=dev)
    sb = res.get("skipbits") if skipbits else None
    head = [ctypes.byref(batch.c), _ptr(q, torch.bfloat16, "q"), _ptr(k_pages, torch.bfloat16, "k_pages"),
            _ptr(v_pages, torch.bfloat16, "v_pages"), _ptr(page_table, torch.int32, "page_table"),
            _ptr(order, torch.int32, "order"), _ptr(count, torch.int32, "count"), int(kmax)]
    if keep is not None:
        head.append(_ptr(keep, torch.uint8, "keep"))
    rc = getattr(_lib(), entry)(
        *head, ctypes.c_float(thr),
        _ptr(res["out"], torch.bfloat16, "out"), _ptr(res["visited"], torch.int32, "visited"),
        _ptr(res["skipped"], torch.int32, "skipped"), _ptr(sb, torch.uint8, "skipbits"),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream())
    _check(rc, entry)
    return res


def attn(batch: Batch, q, k_pages, v_pages, page_table, order, count, kmax: int, tau: float, workspace,
         out=None, skipbits: bool = False):
    """OSK attention with one skip threshold tau.  Returns dict(out, visited, skipped[, skipbits])."""
    return _attn("cosa_attn", batch, q, k_pages, v_pages, page_table, order, count, kmax, tau, workspace, out,
                 skipbits)


def attn_delta(batch: Batch, q, k_pages, v_pages, page_table, order, count, kmax: int, delta: float, workspace,
               out=None, skipbits: bool = False):
    """OSK attention with tau_s = delta / L_s per sequence (delta = -1: no skip)."""
    return _attn("cosa_attn_delta", batch, q, k_pages, v_pages, page_table, order, count, kmax, delta, workspace,
                 out, skipbits)


def attn_masked(batch: Batch, q, k_pages, v_pages, page_table, order, count, kmax: int, keep, tau: float,
                workspace, out=None, skipbits: bool = False):
    """OSK attention in logical-mask execution: every list entry is walked and
    only those with keep[h, I, t] != 0 are computed (the ablation of physical
    jumping over pages)."""
    return _attn("cosa_attn_masked", batch, q, k_pages, v_pages, page_table, order, count, kmax, tau, workspace,
                 out, skipbits, keep=keep)


def check(workspace):
    """Synchronise the current stream and raise CosaError if a kernel reported an error."""
    _check(_lib().cosa_sync_status(_ptr(workspace, torch.uint8, "workspace"), _stream()), "device status")


def set_wait_limit(spins: int):
    """Failure-detection hook: cap pipeline waits of later attn calls (0 = default)."""
    _lib().cosa_debug_set_wait_limit(int(spins))

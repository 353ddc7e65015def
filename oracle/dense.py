"""Brute-force dense causal softmax attention in fp64.

"CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed
Sparse Attention", §3.1 Dense Attention (heading only on the pages; the
standard definition): O = softmax(Q K^T / sqrt(d) + causal mask) V per query
head, with GQA sharing of kv head floor(h / G).  Computed as one full score
matrix per head with a plain softmax -- no blocking, no online rescaling --
so it shares no step with the OSK oracle it is used to check.
"""

from __future__ import annotations

import math

import numpy as np

from ._bf16 import f32


def dense_causal(q_bits, k_pages_bits, v_pages_bits, page_table, seqlens, num_kv_heads,
                 heads=None, rows=None):
    """Dense causal attention over a packed batch, fp64 [T, Hq, d].

    rows: optional per-sequence list of local query-row index arrays (default all).
    Entries not computed are NaN.
    """
    T, Hq, d = q_bits.shape
    G = Hq // num_kv_heads
    b_p = k_pages_bits.shape[2]
    out = np.full((T, Hq, d), np.nan)
    heads = range(Hq) if heads is None else heads
    tok0 = 0
    for s, L in enumerate(seqlens):
        # token p of sequence s: page page_table[s, p // b_p], slot p % b_p
        pos = np.arange(L)
        pages = page_table[s, pos // b_p].astype(np.int64)
        slots = pos % b_p
        r = np.arange(L) if rows is None else np.asarray(rows[s])
        for h in heads:
            kv = h // G
            K = f32(k_pages_bits[pages, kv, slots]).astype(np.float64)   # [L, d]
            V = f32(v_pages_bits[pages, kv, slots]).astype(np.float64)
            Q = f32(q_bits[tok0 + r, h]).astype(np.float64)               # [nr, d]
            S = Q @ K.T / math.sqrt(d)
            S[pos[None, :] > r[:, None]] = -np.inf
            S -= S.max(axis=1, keepdims=True)
            P = np.exp(S)
            P /= P.sum(axis=1, keepdims=True)
            out[tok0 + r, h] = P @ V
        tok0 += L
    return out

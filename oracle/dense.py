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
                 heads=None, rows=None, q_lens=None):
    """Dense causal attention over a packed batch, fp64 [Tq, Hq, d].

    q_lens: per-sequence query counts after a cached prefix (default: every
    token is a query); query t of sequence s sits at position L_s - Lq_s + t
    and attends to keys 0 .. L_s - Lq_s + t.
    rows: optional per-sequence list of local query-row index arrays (default all).
    Entries not computed are NaN.
    """
    Tq, Hq, d = q_bits.shape
    G = Hq // num_kv_heads
    b_p = k_pages_bits.shape[2]
    out = np.full((Tq, Hq, d), np.nan)
    heads = range(Hq) if heads is None else heads
    q_lens = seqlens if q_lens is None else q_lens
    tq0 = 0
    for s, L in enumerate(seqlens):
        Lq = int(q_lens[s])
        off = L - Lq
        # token p of sequence s: page page_table[s, p // b_p], slot p % b_p
        pos = np.arange(L)
        pages = page_table[s, pos // b_p].astype(np.int64)
        slots = pos % b_p
        r = np.arange(Lq) if rows is None else np.asarray(rows[s])
        for h in heads:
            kv = h // G
            K = f32(k_pages_bits[pages, kv, slots]).astype(np.float64)   # [L, d]
            V = f32(v_pages_bits[pages, kv, slots]).astype(np.float64)
            Q = f32(q_bits[tq0 + r, h]).astype(np.float64)               # [nr, d]
            S = Q @ K.T / math.sqrt(d)
            S[pos[None, :] > off + r[:, None]] = -np.inf
            S -= S.max(axis=1, keepdims=True)
            P = np.exp(S)
            P /= P.sum(axis=1, keepdims=True)
            out[tq0 + r, h] = P @ V
        tq0 += Lq
    return out

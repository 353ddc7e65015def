"""Ordered-Skipping Kernel (OSK) oracle: what the kernel computes, step by step, in fp64.

Follows "CoSA: Accelerating Long-Context Inference via Proxy-Kernel
Co-Designed Sparse Attention":
  §3.2       -- online softmax is order invariant (P2): blocks may be visited
                in any order.
  §3.3       -- the in-kernel skip decides on real logits, so S = Q K^T is
                formed for every visited block and only the value side
                (exp, row sum, P V) is trimmed (L1); it compares against a
                running max (L2.1) and is an AND over rows (L2.2).
  §4.3       -- OSK visits only the retained pages, in M_KAP order, and skips
                per 128-row query tile with one tile-wide vote.
  Appendix C.2 / Algorithm A -- traverse the retained pages in order, update
                the online-softmax statistics from exact logits, skip the
                value side when the criterion holds.
  Appendix D.1 -- logical blocks of b tokens; the vote reuses the row maxima
                the online softmax already keeps.

Reading of the missing Eq. (5): for a visited block with logits
s_rt = q_r . k_t / sqrt(d) (causal and sequence-end masks applied),
m~_r = max_t s_rt; delta = max over the tile's valid rows of (m~_r - m_r)
with m_r the running max before the block; the block's value side is
skipped iff delta < ln(tau).  tau = 0 never skips; the first visited block
(m = -inf) is never skipped; a skipped block changes none of m, l, O.
"""

from __future__ import annotations

import math

import numpy as np

from ._bf16 import f32, gather_tokens
from ._layout import query_blocks


def osk_tile(qrows, qpos, blocks, order, tau, scale):
    """One (head, q-block) tile.

    qrows: fp64 [nr, d] valid query rows; qpos: absolute positions [nr].
    blocks(j) -> (K fp64 [nk, d], V fp64 [nk, d], kpos [nk]) for key block j.
    order: key block indices in visit order.
    Returns (out fp64 [nr, d], skipped bool [len(order)], delta fp64 [len(order)]).
    """
    nr, d = qrows.shape
    log_tau = math.log(tau) if tau > 0 else -math.inf
    m = np.full(nr, -np.inf)
    l = np.zeros(nr)
    O = np.zeros((nr, d))
    skipped = np.zeros(len(order), dtype=bool)
    deltas = np.zeros(len(order))
    for t, j in enumerate(order):
        K, V, kpos = blocks(int(j))
        S = (qrows @ K.T) * scale
        S = np.where(kpos[None, :] <= qpos[:, None], S, -np.inf)      # causal
        m_blk = S.max(axis=1)
        with np.errstate(invalid="ignore"):
            gap = np.where(np.isneginf(m_blk), -np.inf, m_blk - m)     # m = -inf -> +inf
        delta = float(gap.max())
        deltas[t] = delta
        if delta < log_tau:
            skipped[t] = True
            continue
        m_new = np.maximum(m, m_blk)
        with np.errstate(invalid="ignore"):
            alpha = np.where(np.isneginf(m), 0.0, np.exp(m - m_new))
        base = np.where(np.isneginf(m_new), 0.0, m_new)
        P = np.exp(S - base[:, None])
        l = l * alpha + P.sum(axis=1)
        O = O * alpha[:, None] + P @ V
        m = m_new
    return O / l[:, None], skipped, deltas


class PagedSequence:
    """Logical fp64 view of one sequence's K/V for one kv head in the page pool (oracle's own gather)."""

    def __init__(self, k_pages_bits, v_pages_bits, table_row, length, block_size, kv_head):
        self.k = f32(gather_tokens(k_pages_bits[:, kv_head:kv_head + 1], table_row, length)[:, 0]).astype(np.float64)
        self.v = f32(gather_tokens(v_pages_bits[:, kv_head:kv_head + 1], table_row, length)[:, 0]).astype(np.float64)
        self.length = length
        self.b = block_size

    def block(self, j):
        lo, hi = j * self.b, min(self.length, (j + 1) * self.b)
        return self.k[lo:hi], self.v[lo:hi], np.arange(lo, hi)


def osk_units(q_bits, k_pages_bits, v_pages_bits, page_table, seqlens, num_kv_heads, block_size,
              order, count, tau, units=None, q_lens=None):
    """OSK tile by tile: yields (h, I, rows, out, skipped, delta) for each (h, I) unit.

    rows: the unit's slice of the packed query rows; out fp64 [rows, d];
    skipped bool / delta fp64 [count[h, I]] in visit order.  Arguments as in osk().
    Units are visited grouped by (sequence, kv head), so that one gathered view
    of a sequence's keys and values serves all of its units.
    """
    Tq, Hq, d = q_bits.shape
    G = Hq // num_kv_heads
    b = block_size
    scale = 1.0 / math.sqrt(d)
    NQB = order.shape[1]
    layout = query_blocks(seqlens, q_lens, b)
    taus = list(tau) if np.ndim(tau) else [tau] * len(seqlens)
    seq_of = np.concatenate([np.full(nb - i0, s) for s, (_, i0, nb, _) in enumerate(layout)])
    blk0 = np.concatenate([[0], np.cumsum([nb - i0 for _, i0, nb, _ in layout])])
    if units is None:
        units = [(h, I) for h in range(Hq) for I in range(NQB)]
    units = sorted(set((int(h), int(I)) for h, I in units), key=lambda u: (seq_of[u[1]], u[0] // G, u))
    key, seq = None, None
    for h, I in units:
        s = int(seq_of[I])
        if key != (s, h // G):
            key = (s, h // G)
            seq = PagedSequence(k_pages_bits, v_pages_bits, page_table[s], seqlens[s], b, h // G)
        off, i0, _, tq0 = layout[s]
        i = i0 + I - blk0[s]
        L = seqlens[s]
        r0, r1 = max(off, i * b), min(L, (i + 1) * b)        # absolute positions of the rows
        rows = slice(tq0 + r0 - off, tq0 + r1 - off)          # their place in the packed Q
        qrows = f32(q_bits[rows, h]).astype(np.float64)
        k_i = int(count[h, I])
        o, sk, de = osk_tile(qrows, np.arange(r0, r1), seq.block, order[h, I, :k_i], taus[s], scale)
        yield h, I, rows, o, sk, de


def osk(q_bits, k_pages_bits, v_pages_bits, page_table, seqlens, num_kv_heads, block_size,
        order, count, tau, units=None, q_lens=None):
    """OSK over a packed batch.

    order/count: the proxy's ordered lists [Hq, NQB, kmax] / [Hq, NQB].
    q_lens: per-sequence query counts for prefill after a cached prefix
    (default: every token is a query); query t of sequence s sits at
    position L_s - Lq_s + t, and a tile holds the q-block's present rows.
    tau: one threshold, or a sequence of one per sequence.
    units: optional iterable of (h, I) tiles to compute (default: all).
    Returns dict: out fp64 [Tq, Hq, d] (NaN where not computed), visited and
    skipped int32 [Hq, NQB] (-1 where not computed), skip bool and delta
    fp64 [Hq, NQB, kmax] (padding False / NaN).
    """
    Tq, Hq, d = q_bits.shape
    NQB, kmax = order.shape[1], order.shape[2]
    out = np.full((Tq, Hq, d), np.nan)
    visited = np.full((Hq, NQB), -1, dtype=np.int32)
    skipped = np.full((Hq, NQB), -1, dtype=np.int32)
    skip = np.zeros((Hq, NQB, kmax), dtype=bool)
    delta = np.full((Hq, NQB, kmax), np.nan)
    for h, I, rows, o, sk, de in osk_units(q_bits, k_pages_bits, v_pages_bits, page_table, seqlens, num_kv_heads,
                                           block_size, order, count, tau, units, q_lens):
        k_i = len(sk)
        out[rows, h] = o
        visited[h, I] = k_i
        skipped[h, I] = int(sk.sum())
        skip[h, I, :k_i] = sk
        delta[h, I, :k_i] = de
    return dict(out=out, visited=visited, skipped=skipped, skip=skip, delta=delta)

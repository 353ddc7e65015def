"""Kernel-Aware Proxy (KAP) oracle.

Follows "CoSA: Accelerating Long-Context Inference via Proxy-Kernel
Co-Designed Sparse Attention":
  §4.1 Overview      -- KAP emits an ordered mask M_KAP, HRM ("have rowmax")
                        blocks first, under a moderate stage-1 budget.
  §4.2 KAP design    -- "Block ranking" and "Flag-grouped sorting" (both
                        paragraph bodies are missing from the pages).
  §5.1 Impl. details -- scoring and pooling are one fused kernel.
  Appendix C.1 / Figure A -- every candidate key block gets an importance
                        score and an HRM flag; the HRM and non-HRM groups are
                        sorted independently by score, HRM group first, and
                        the leading entries under the budget are kept.

Readings of what the pages leave open (each one fixed here; the CUDA path
follows the same definitions):
  * Score: pooled QK.  Per q-block the fp32 sum of its query rows, per key
    block the fp32 sum of its valid keys; both quantised to int8 per vector
    (symmetric, max-abs scale, round half to even); the dot product is the
    exact integer sum; score = float32(dot) * ks_j with
    ks_j = (M_j / 127) / n_tok(j).  The query scale is a positive constant
    along a row and is dropped: only the ranking matters.
  * Sums run sequentially over tokens for every dimension; the q-block sum
    is the sequential fold of its sub-row sums.
  * HRM: the q-block is cut into sub-rows of g = 16 query rows; a key block
    is HRM iff it is the argmax (lowest index on ties) of some valid
    sub-row's scores over the candidates j <= i.
  * Candidates of q-block i are its causal key blocks j = 0..i; n_i = i + 1.
  * Budget: bp = floor(budget * 1e4 + 0.5); k_i = max(1, ceil(n_i bp / 1e4)).
  * Order key: (HRM first, score descending, block index ascending); keep the
    first k_i.  No block is forced in.
  * Top-p (the pages' stage-1 rule, §5.1 "Hyperparameters"; the pages give
    p only): block j's mass is n_tok(j) exp(z_j), z_j the mean logit
    estimated from the pooled score; k_i is the shortest prefix of the
    order above whose share of the row's mass reaches p (top_p_count).
"""

from __future__ import annotations

import math

import numpy as np

from ._bf16 import f32, gather_tokens
from ._layout import num_query_blocks, query_blocks

SUB_ROWS = 16          # g: query rows per HRM sub-row
_F127 = np.float32(127.0)
_TINY = np.float32(2.0 ** -126)   # below the smallest normal fp32: vector treated as zero


def budget_bp(budget: float) -> int:
    """Budget fraction -> basis points, rounded half up (in double)."""
    return int(math.floor(float(np.float32(budget)) * 1e4 + 0.5))


def keep_count(n_i: int, bp: int) -> int:
    """k_i = max(1, ceil(n_i * bp / 10^4)) in integers."""
    return max(1, (n_i * bp + 9999) // 10000)


def kmax_for(max_qblocks: int, budget: float) -> int:
    return keep_count(max_qblocks, budget_bp(budget))


def quantize_int8(v: np.ndarray):
    """Symmetric int8 quantisation of each vector along the last axis.

    M = max |v_d|; a vector with M below 2^-126 (zero or subnormal) becomes
    all zeros; otherwise inv = 127 / M (fp32) and q_d = rint(v_d * inv)
    (fp32 product, round half to even).  Returns (q int8, M float32).
    """
    v = np.asarray(v, dtype=np.float32)
    M = np.max(np.abs(v), axis=-1)
    tiny = M < _TINY
    inv = (_F127 / np.where(tiny, np.float32(1.0), M)).astype(np.float32)
    inv = np.where(tiny, np.float32(0.0), inv).astype(np.float32)
    prod = (v * inv[..., None]).astype(np.float32)
    q = np.rint(prod)
    assert np.all(np.abs(q) <= 127)
    return q.astype(np.int8), M.astype(np.float32)


def pool_keys(kf: np.ndarray, length: int, b: int):
    """Per key block j: fp32 sum over its valid tokens, token by token.

    kf: float32 [length, Hkv, d] (logical order).
    Returns (sums float32 [nkb, Hkv, d], ntok int [nkb]).
    """
    nkb = (length + b - 1) // b
    H, d = kf.shape[1], kf.shape[2]
    padded = np.zeros((nkb * b, H, d), dtype=np.float32)
    padded[:length] = kf
    blocks = padded.reshape(nkb, b, H, d)
    ntok = np.array([min(b, length - j * b) for j in range(nkb)], dtype=np.int64)
    acc = np.zeros((nkb, H, d), dtype=np.float32)
    for t in range(b):
        valid = ntok > t                               # token t exists in block j
        acc[valid] = (acc[valid] + blocks[valid, t]).astype(np.float32)
    return acc, ntok


def quantize_keys(sums: np.ndarray, ntok: np.ndarray):
    """int8 key vectors and fp32 scale ks_j = (M_j / 127) / n_tok(j) (0 if M tiny)."""
    k8, M = quantize_int8(sums)                       # [nkb, Hkv, d], [nkb, Hkv]
    ks = ((M / _F127).astype(np.float32) / ntok.astype(np.float32)[:, None]).astype(np.float32)
    ks = np.where(M < _TINY, np.float32(0.0), ks).astype(np.float32)
    return k8, ks


def pool_queries(qf: np.ndarray, length: int, b: int, g: int = SUB_ROWS, offset: int = 0):
    """Per q-block: the fp32 sums of its R = b/g sub-rows and of the whole block.

    qf: float32 [length, Hq, d] by absolute position; the rows at positions
    below `offset` (a cached prefix) are absent and never read.  A row is
    valid iff offset <= position < length.  A sub-row sums its valid rows one
    by one; a sub-row with no valid row sums to +0 and is invalid.  The block
    sum folds the R sub-row sums in order starting from +0.
    Returns (sub float32 [nqb, R, Hq, d], blk float32 [nqb, Hq, d],
             sub_valid bool [nqb, R]).
    """
    nqb = (length + b - 1) // b
    R = b // g
    H, d = qf.shape[1], qf.shape[2]
    padded = np.zeros((nqb * b, H, d), dtype=np.float32)
    padded[:length] = qf
    rows = padded.reshape(nqb, R, g, H, d)
    first_row = (np.arange(nqb)[:, None] * b + np.arange(R)[None, :] * g)   # [nqb, R]
    sub = np.zeros((nqb, R, H, d), dtype=np.float32)
    for t in range(g):
        valid = ((first_row + t) < length) & ((first_row + t) >= offset)
        sub[valid] = (sub[valid] + rows[:, :, t][valid]).astype(np.float32)
    blk = np.zeros((nqb, H, d), dtype=np.float32)
    for r in range(R):
        blk = (blk + sub[:, r]).astype(np.float32)
    return sub, blk, (first_row < length) & (first_row + g > offset)


def int_dots(a8: np.ndarray, b8: np.ndarray) -> np.ndarray:
    """Exact integer dot products a8 @ b8.T (int8 inputs) as int64.

    Every partial sum is an integer of magnitude < 2^53, so the fp64 matrix
    product is exact whatever order the library sums in.
    """
    return np.rint(a8.astype(np.float64) @ b8.astype(np.float64).T).astype(np.int64)


def scores_from_dots(dots: np.ndarray, ks: np.ndarray) -> np.ndarray:
    """score = float32(dot) * ks_j, one fp32 rounding."""
    return (dots.astype(np.float32) * ks.astype(np.float32)).astype(np.float32)


def select_row(score: np.ndarray, sub_scores: np.ndarray, sub_valid: np.ndarray, k_i: int):
    """Flag-grouped selection for one (head, q-block) row.

    score: float32 [n_i] block scores over candidates j = 0..i;
    sub_scores: float32 [R, n_i]; sub_valid: bool [R].
    Returns (order int [k_i], hrm bool [k_i], hrm_all bool [n_i]).
    """
    n_i = score.shape[0]
    hrm = np.zeros(n_i, dtype=bool)
    for r in range(sub_scores.shape[0]):
        if sub_valid[r]:
            hrm[int(np.argmax(sub_scores[r]))] = True     # first maximum = lowest j
    j = np.arange(n_i)
    # lexsort: last key is primary.  HRM first, score descending, j ascending.
    idx = np.lexsort((j, -score.astype(np.float64), ~hrm))
    order = idx[:k_i]
    return order, hrm[order], hrm


def _scored_rows(q_bits, k_pages_bits, page_table, seqlens, num_kv_heads, block_size, g,
                 heads, q_lens):
    """Every (query head h, list row I) of a packed batch with what its selection needs.

    Yields (h, I, i, s_blk [n_i], s_sub [R, n_i], sub_valid [R], ntok [n_i],
    M_q, n_rows): block and sub-row scores over the candidates j = 0..i, the
    key blocks' token counts, the q-block sum's max-abs and its number of
    query rows.  q_lens as in oracle._layout.query_blocks.
    """
    Hq = q_bits.shape[1]
    G = Hq // num_kv_heads
    b = block_size
    heads = range(Hq) if heads is None else heads
    I0 = 0
    for s, (off, i0, nqb, tq0) in enumerate(query_blocks(seqlens, q_lens, b)):
        L = int(seqlens[s])
        kf = f32(gather_tokens(k_pages_bits, page_table[s], L))
        ksum, ntok = pool_keys(kf, L, b)
        k8, ks = quantize_keys(ksum, ntok)
        qf = np.zeros((L,) + q_bits.shape[1:], dtype=np.float32)
        qf[off:] = f32(q_bits[tq0:tq0 + L - off])      # query t at position off + t
        sub, blk, sub_valid = pool_queries(qf, L, b, g, off)
        q8_sub, _ = quantize_int8(sub)     # [nqb, R, Hq, d]
        q8_blk, Mq = quantize_int8(blk)    # [nqb, Hq, d], [nqb, Hq]
        R = sub.shape[1]
        for h in heads:
            kv = h // G
            s_blk = scores_from_dots(int_dots(q8_blk[:, h], k8[:, kv]), ks[:, kv])       # [nqb, nkb]
            s_sub = scores_from_dots(int_dots(q8_sub[:, :, h].reshape(nqb * R, -1), k8[:, kv]),
                                     ks[:, kv]).reshape(nqb, R, nqb)
            for i in range(i0, nqb):
                n_rows = min(L, (i + 1) * b) - max(off, i * b)
                yield (h, I0 + i - i0, i, s_blk[i, :i + 1], s_sub[i, :, :i + 1], sub_valid[i],
                       ntok[:i + 1], float(Mq[i, h]), n_rows)
        I0 += nqb - i0


def kap_proxy(q_bits, k_pages_bits, page_table, seqlens, num_kv_heads, block_size, budget,
              g: int = SUB_ROWS, kmax: int | None = None, heads=None, q_lens=None):
    """KAP over a packed batch.

    q_lens: per-sequence query counts for prefill after a cached prefix
    (default: every token is a query); q_bits then holds only those rows.
    Returns dict with order int32 [Hq, NQB, kmax] (-1 pad; NQB = the present
    q-blocks), count int32 [Hq, NQB], n_hrm int32 [Hq, NQB], hrm uint8
    [Hq, NQB, kmax], kmax.
    `heads` restricts the work to a subset of query heads (others stay -1/0).
    """
    Hq = q_bits.shape[1]
    b = block_size
    bp = budget_bp(budget)
    NQB = num_query_blocks(seqlens, q_lens, b)
    if kmax is None:
        kmax = keep_count(max((L + b - 1) // b for L in seqlens), bp)
    order = np.full((Hq, NQB, kmax), -1, dtype=np.int32)
    hrm_out = np.zeros((Hq, NQB, kmax), dtype=np.uint8)
    count = np.zeros((Hq, NQB), dtype=np.int32)
    n_hrm = np.zeros((Hq, NQB), dtype=np.int32)
    for h, I, i, s_blk, s_sub, sub_valid, _, _, _ in _scored_rows(
            q_bits, k_pages_bits, page_table, seqlens, num_kv_heads, b, g, heads, q_lens):
        k_i = keep_count(i + 1, bp)
        o, fl, _ = select_row(s_blk, s_sub, sub_valid, k_i)
        order[h, I, :k_i] = o
        hrm_out[h, I, :k_i] = fl
        count[h, I] = k_i
        n_hrm[h, I] = int(fl.sum())
    return dict(order=order, count=count, n_hrm=n_hrm, hrm=hrm_out, kmax=kmax)


def top_p_count(ordered_scores: np.ndarray, ordered_ntok: np.ndarray, zscale: float, p: float,
                eps: float = 1e-6):
    """Stage-1 Top-p cut of one row (§5.1 "Hyperparameters", Appendix D.1: the
    pages fix p, not the mass; this is the reading of this build).

    ordered_scores: float32 [n_i] pooled scores of the candidates, already in
    the visit order (HRM first, score descending, block index ascending);
    ordered_ntok: their token counts; zscale > 0 turns a pooled score into the
    mean logit between the q-block's rows and the block's keys:
      z_j = score_j * zscale,  zscale = (M_q / 127) / (n_rows * sqrt(d)),
    with M_q the q-block sum's quantisation scale (dropped from the ranking
    score, needed for a mass).  Block j's share of the row's attention is
      w_j = n_tok(j) exp(z_j - max z) / sum_j' n_tok(j') exp(z_j' - max z)
    (fp64).  k = the shortest prefix of the order whose share is >= p (at
    least 1); p = 1 keeps the whole list, as it does in exact arithmetic
    even where a far tail's fp64 mass underflows to zero.  Also returned: the window
    [k_lo, k_hi] of prefix lengths whose share lies within eps of p, where a
    computation in another precision may legitimately cut instead.
    Returns (k, k_lo, k_hi).
    """
    if not 0.0 < p <= 1.0:
        raise ValueError("p must lie in (0, 1]")
    z = ordered_scores.astype(np.float64) * float(zscale)
    mass = ordered_ntok.astype(np.float64) * np.exp(z - z.max())
    cum = np.cumsum(mass)
    share = cum / cum[-1]
    share[-1] = 1.0
    n = share.shape[0]
    if p >= 1.0:
        return n, n, n            # every mass is positive: only the whole list reaches 1
    k = int(np.searchsorted(share, p, side="left")) + 1     # first prefix with share >= p
    k = min(max(k, 1), n)
    near = np.nonzero(np.abs(share - p) <= eps)[0]
    k_lo = min(k, int(near.min()) + 1) if near.size else k
    k_hi = max(k, int(near.max()) + 2) if near.size else k
    return k, k_lo, min(k_hi, n)


def kap_proxy_top_p(q_bits, k_pages_bits, page_table, seqlens, num_kv_heads, block_size, p: float,
                    g: int = SUB_ROWS, eps: float = 1e-6, q_lens=None):
    """KAP with the Top-p stage-1 cut instead of a budget fraction.

    Same scores, HRM flags and order as kap_proxy; each row keeps the
    top_p_count prefix of its full flag-grouped order, with
    zscale = (M_q / 127) / (n_rows sqrt(d)).  Returns dict with order int32
    [Hq, NQB, kmax] (kmax = the longest sequence's block count, -1 pad),
    count, count_lo, count_hi int32 [Hq, NQB] (the cut and its eps window),
    n_hrm, hrm.
    """
    Hq, d = q_bits.shape[1], q_bits.shape[2]
    b = block_size
    NQB = num_query_blocks(seqlens, q_lens, b)
    kmax = max((L + b - 1) // b for L in seqlens)
    order = np.full((Hq, NQB, kmax), -1, dtype=np.int32)
    hrm_out = np.zeros((Hq, NQB, kmax), dtype=np.uint8)
    count = np.zeros((Hq, NQB), dtype=np.int32)
    count_lo = np.zeros((Hq, NQB), dtype=np.int32)
    count_hi = np.zeros((Hq, NQB), dtype=np.int32)
    n_hrm = np.zeros((Hq, NQB), dtype=np.int32)
    for h, I, i, s_blk, s_sub, sub_valid, ntok, Mq, n_rows in _scored_rows(
            q_bits, k_pages_bits, page_table, seqlens, num_kv_heads, b, g, None, q_lens):
        o, fl, _ = select_row(s_blk, s_sub, sub_valid, i + 1)
        zscale = (Mq / 127.0) / (n_rows * math.sqrt(d))
        k, k_lo, k_hi = top_p_count(s_blk[o], ntok[o], zscale, p, eps)
        order[h, I, :k] = o[:k]
        hrm_out[h, I, :k] = fl[:k]
        count[h, I], count_lo[h, I], count_hi[h, I] = k, k_lo, k_hi
        n_hrm[h, I] = int(fl[:k].sum())
    return dict(order=order, count=count, count_lo=count_lo, count_hi=count_hi, n_hrm=n_hrm, hrm=hrm_out,
                kmax=kmax)


def remap(order, count, page_table, seqlens, block_size, page_size, q_lens=None):
    """Ordered key blocks -> physical pages, page by page (§4.3 "Any-order page visiting").

    pages[h, I, t * ppb + u] = page_table[s, order[h, I, t] * ppb + u] when
    t < count[h, I] and that logical page holds tokens of sequence s
    (order * b + u * b_p < L_s); -1 otherwise.  ppb = b / b_p.
    """
    Hq, NQB, kmax = order.shape
    ppb = block_size // page_size
    out = np.full((Hq, NQB, kmax * ppb), -1, dtype=np.int32)
    t = np.arange(kmax)
    blk0 = 0
    for s, (_, i0, nb, _) in enumerate(query_blocks(seqlens, q_lens, block_size)):
        L = int(seqlens[s])
        nqb = nb - i0                                               # this sequence's list rows
        o = order[:, blk0:blk0 + nqb, :].astype(np.int64)            # [Hq, nqb, kmax]
        listed = t[None, None, :] < count[:, blk0:blk0 + nqb, None]
        for u in range(ppb):
            inside = listed & (o >= 0) & (o * block_size + u * page_size < L)
            logical = np.where(inside, o * ppb + u, 0)
            out[:, blk0:blk0 + nqb, u::ppb] = np.where(inside, page_table[s][logical], -1)
        blk0 += nqb
    return out

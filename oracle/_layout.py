"""Query-block layout of a packed batch, for prefill with or without a cached prefix.

"CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed
Sparse Attention" treats prefill (every token of the sequence is a query) and
names integration with paged-KV serving frameworks (§4.3, Appendix D.1).
With a cached prefix (q_len < kv_len) the pages are silent; the reading fixed
here: sequence s has L_s keys and its last Lq_s tokens are the queries, so
query t sits at absolute position off_s + t, off_s = L_s - Lq_s.  Logical
q-blocks stay on the kv block grid: q-block i covers absolute positions
[i b, (i + 1) b) intersected with [off_s, L_s), its candidates are the key
blocks j = 0..i, and the q-blocks wholly inside the prefix do not exist.
The first present q-block i0 = floor(off_s / b) may lack its leading rows.
"""

from __future__ import annotations


def query_blocks(seqlens, q_lens, b):
    """Per sequence (off, i0, nb, tq0): prefix length, first present q-block,
    number of kv blocks, and the sequence's first row in the packed Q.

    q_lens None means q_len = kv_len for every sequence.  Requires
    1 <= Lq_s <= L_s.
    """
    if q_lens is None:
        q_lens = seqlens
    if len(q_lens) != len(seqlens):
        raise ValueError("q_lens and seqlens differ in length")
    out = []
    tq0 = 0
    for L, Lq in zip(seqlens, q_lens):
        L, Lq = int(L), int(Lq)
        if not 1 <= Lq <= L:
            raise ValueError("need 1 <= q_len <= kv_len")
        off = L - Lq
        out.append((off, off // b, (L + b - 1) // b, tq0))
        tq0 += Lq
    return out


def num_query_blocks(seqlens, q_lens, b):
    """Rows of the ordered lists: the present q-blocks of all sequences."""
    return sum(nb - i0 for _, i0, nb, _ in query_blocks(seqlens, q_lens, b))

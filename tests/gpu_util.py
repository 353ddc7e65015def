"""Shared helpers of the GPU parity tests: upload a workload, run the library
through its C ABI, compare against the oracle with the stated tolerances.

Tolerances (bf16 outputs of the attention): max-abs 2e-2 and mean-abs 2e-3
against the oracle's fp64 result; skip sets identical except blocks whose
oracle statistic delta lies within 1e-3 of ln(tau).  Block lists, counts, HRM
flags and page lists: bit-exact.
"""

from __future__ import annotations

import math

import numpy as np
import torch

import block_sparse_long_14_b200 as cosa

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
DELTA_WINDOW = 1e-3


def prefix_q(w, q_lens):
    """Packed Q of prefill after a cached prefix: each sequence's last q_len rows."""
    parts, tok0 = [], 0
    for L, Lq in zip(w.seqlens, q_lens):
        parts.append(w.q[tok0 + L - Lq:tok0 + L])
        tok0 += L
    return np.ascontiguousarray(np.concatenate(parts, axis=0))


def upload(w, device="cuda", q_lens=None):
    """Device copies of a workload; with q_lens, only the query rows of Q."""
    def bf16(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(device)

    batch = cosa.Batch(w.seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.page_size,
                       w.num_pages, w.max_pages_per_seq, device=device, q_lens=q_lens)
    q = w.q if q_lens is None else prefix_q(w, q_lens)
    return dict(batch=batch, q=bf16(q), k_pages=bf16(w.k_pages), v_pages=bf16(w.v_pages),
                page_table=torch.from_numpy(np.ascontiguousarray(w.page_table)).to(device))


def run_proxy(d, budget):
    ws, kmax = cosa.alloc_workspace(d["batch"], budget)
    sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], budget, kmax, ws)
    cosa.check(ws)
    return {k: v.cpu().numpy() for k, v in sel.items()}, kmax, ws


def run_attn(d, sel_dev, kmax, tau, ws):
    res = cosa.attn(d["batch"], d["q"], d["k_pages"], d["v_pages"], d["page_table"], sel_dev["order"],
                    sel_dev["count"], kmax, tau, ws, skipbits=True)
    cosa.check(ws)
    return res


def assert_proxy_equal(got, ref, rows=None):
    """Bit-exact comparison of the proxy outputs (optionally on (h, I) rows only)."""
    for key in ("order", "count", "n_hrm", "hrm"):
        g, r = got[key], ref[key]
        if rows is not None:
            g = g[rows[:, 0], rows[:, 1]]
            r = r[rows[:, 0], rows[:, 1]]
        if not np.array_equal(g, r):
            bad = np.argwhere(g != r)
            raise AssertionError(f"proxy {key} differs at {len(bad)} places, first {bad[:5].tolist()}: "
                                 f"gpu {g[tuple(bad[0])]} vs oracle {r[tuple(bad[0])]}")


def _max_abs_v(w):
    """max |V| over the page pool, from the bf16 bit patterns (sign bit cleared)."""
    top = int(np.max(np.asarray(w.v_pages).view(np.uint16) & np.uint16(0x7FFF)))
    return float(np.array([top << 16], dtype=np.uint32).view(np.float32)[0])


def _unit_ref(ref, h, I, rows):
    """(out rows, visited, skip, delta) of one tile, from the oracle's full result
    dict or from OraclePool.run's per-tile dict."""
    if isinstance(ref, dict) and "out" in ref:
        k = int(ref["visited"][h, I])
        return ref["out"][rows, h], k, ref["skip"][h, I, :k], ref["delta"][h, I, :k]
    r, o, sk, de = ref[(h, I)]
    assert (r.start, r.stop) == (rows.start, rows.stop), f"unit ({h},{I}): oracle rows {r} vs {rows}"
    return o, len(sk), sk, de


def compare_attn(res, ref, w, tau, units, q_lens=None):
    """Compare GPU OSK results with the oracle on the given (h, I) units.

    ref: the oracle's result dict (osk.osk) or OraclePool.run's per-tile dict.
    q_lens: per-sequence query counts of prefill after a cached prefix (rows
    and list rows then cover only the queries).

    Skip decisions must match except for blocks whose oracle statistic delta
    lies within DELTA_WINDOW of ln(tau).  A unit with such a flipped decision is
    still compared element by element: each flipped block moves a row by at
    most 2 b tau e^DELTA_WINDOW max|V| (its keys weigh below about tau against
    the running max, and the row sum is at least 1 in those units), which is
    added to the unit's max-abs tolerance.  Every unit's skipped count must
    equal the number of skip bits the kernel itself set.
    Returns a dict of statistics; raises AssertionError on a violation.
    """
    out = res["out"].float().cpu().numpy()
    visited = res["visited"].cpu().numpy()
    skipped = res["skipped"].cpu().numpy()
    skipbits = res["skipbits"].cpu().numpy().astype(bool)
    b = w.block_size
    log_tau = math.log(tau) if tau > 0 else -math.inf
    q_lens = list(w.seqlens) if q_lens is None else list(q_lens)
    seq_of, tok0, nq = [], [0], []
    for s, (L, Lq) in enumerate(zip(w.seqlens, q_lens)):
        nq.append((L + b - 1) // b - (L - Lq) // b)           # q-blocks holding a query row
        seq_of += [s] * nq[-1]
        tok0.append(tok0[-1] + Lq)
    blk0 = np.concatenate([[0], np.cumsum(nq)])
    errs, n_el, max_err, exempt_units, n_skip, n_flip_total = 0.0, 0, 0.0, 0, 0, 0
    exempt_max, vmax = 0.0, None
    for h, I in units:
        s = seq_of[I]
        L = w.seqlens[s]
        off = L - q_lens[s]
        i = I - blk0[s] + off // b
        rows = slice(tok0[s] + max(off, i * b) - off, tok0[s] + min(L, (i + 1) * b) - off)
        ref_out, k, ref_skip, ref_delta = _unit_ref(ref, h, I, rows)
        assert visited[h, I] == k, f"visited[{h},{I}] {visited[h, I]} != {k}"
        gs = skipbits[h, I, :k]
        assert not skipbits[h, I, k:].any()
        assert skipped[h, I] == int(gs.sum()), f"skipped[{h},{I}] {skipped[h, I]} != {int(gs.sum())} skip bits"
        diff = gs != ref_skip
        n_flip = int(diff.sum())
        if n_flip:
            dl = ref_delta[diff]
            assert np.all(np.abs(dl - log_tau) <= DELTA_WINDOW), (
                f"unit ({h},{I}): skip decisions differ at {np.flatnonzero(diff).tolist()} with oracle delta "
                f"{dl.tolist()} vs ln tau {log_tau}")
            exempt_units += 1
            n_flip_total += n_flip
        n_skip += int(gs.sum())
        got = out[rows, h]
        assert np.isfinite(got).all(), f"unit ({h},{I}): non-finite output"
        e = np.abs(got.astype(np.float64) - ref_out)
        if n_flip:
            if vmax is None:
                vmax = _max_abs_v(w)
            allow = MAX_ABS + n_flip * 2.0 * b * tau * math.exp(DELTA_WINDOW) * vmax
            assert e.max() <= allow, f"unit ({h},{I}): max-abs {e.max()} above {allow} with {n_flip} flipped blocks"
            exempt_max = max(exempt_max, float(e.max()))
        else:
            max_err = max(max_err, float(e.max()))
        errs += float(e.sum())
        n_el += e.size
    assert exempt_units <= max(1, len(units) // 100), f"{exempt_units} units with exempt skip differences"
    mean = errs / max(1, n_el)
    assert max_err <= MAX_ABS, f"max-abs {max_err}"
    assert mean <= MEAN_ABS, f"mean-abs {mean}"
    return dict(max_abs=max_err, mean_abs=mean, units=len(units), exempt_units=exempt_units,
                flipped_blocks=n_flip_total, exempt_max_abs=exempt_max, skipped=n_skip)


def all_units(w):
    return [(h, I) for h in range(w.num_q_heads) for I in range(sum((L + w.block_size - 1) // w.block_size
                                                                     for L in w.seqlens))]


def sample_units(w, n, seed=0):
    """A seeded sample of n (h, I) tiles that always includes each sequence's first
    and last q-block (for every head when n allows)."""
    rng = np.random.default_rng(seed)
    b = w.block_size
    nqb = [(L + b - 1) // b for L in w.seqlens]
    blk0 = np.concatenate([[0], np.cumsum(nqb)])
    edges = sorted({int(I) for s in range(len(w.seqlens)) for I in (blk0[s], blk0[s + 1] - 1)})
    units = set()
    if len(edges) * w.num_q_heads <= n:
        units.update((h, I) for I in edges for h in range(w.num_q_heads))
    else:
        units.update((int(rng.integers(w.num_q_heads)), I) for I in edges)
    total = int(blk0[-1])
    while len(units) < n:
        units.add((int(rng.integers(w.num_q_heads)), int(rng.integers(total))))
    return sorted(units)

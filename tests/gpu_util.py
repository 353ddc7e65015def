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


def compare_attn(res, ref, w, tau, units, q_lens=None):
    """Compare GPU OSK results with the oracle on the given (h, I) units.

    q_lens: per-sequence query counts of prefill after a cached prefix (rows
    and list rows then cover only the queries).
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
    errs, n_el, max_err, exempt_units, n_skip = 0.0, 0, 0.0, 0, 0
    for h, I in units:
        s = seq_of[I]
        L = w.seqlens[s]
        off = L - q_lens[s]
        i = I - blk0[s] + off // b
        k = int(ref["visited"][h, I])
        assert visited[h, I] == k, f"visited[{h},{I}] {visited[h, I]} != {k}"
        gs, rs = skipbits[h, I, :k], ref["skip"][h, I, :k]
        assert not skipbits[h, I, k:].any()
        diff = gs != rs
        if diff.any():
            dl = ref["delta"][h, I, :k][diff]
            assert np.all(np.abs(dl - log_tau) <= DELTA_WINDOW), (
                f"unit ({h},{I}): skip decisions differ at {np.flatnonzero(diff).tolist()} with oracle delta "
                f"{dl.tolist()} vs ln tau {log_tau}")
            exempt_units += 1
            continue
        assert skipped[h, I] == int(gs.sum())
        n_skip += int(gs.sum())
        rows = slice(tok0[s] + max(off, i * b) - off, tok0[s] + min(L, (i + 1) * b) - off)
        e = np.abs(out[rows, h].astype(np.float64) - ref["out"][rows, h])
        assert np.isfinite(out[rows, h]).all()
        max_err = max(max_err, float(e.max()))
        errs += float(e.sum())
        n_el += e.size
    assert exempt_units <= max(1, len(units) // 100), f"{exempt_units} units with exempt skip differences"
    mean = errs / max(1, n_el)
    assert max_err <= MAX_ABS, f"max-abs {max_err}"
    assert mean <= MEAN_ABS, f"mean-abs {mean}"
    return dict(max_abs=max_err, mean_abs=mean, units=len(units), exempt_units=exempt_units, skipped=n_skip)


def all_units(w):
    return [(h, I) for h in range(w.num_q_heads) for I in range(sum((L + w.block_size - 1) // w.block_size
                                                                     for L in w.seqlens))]


def sample_units(w, n, seed=0):
    """A seeded sample of (h, I) tiles that always includes each sequence's first and last q-block."""
    rng = np.random.default_rng(seed)
    b = w.block_size
    nqb = [(L + b - 1) // b for L in w.seqlens]
    blk0 = np.concatenate([[0], np.cumsum(nqb)])
    units = set()
    for s in range(len(w.seqlens)):
        for I in (blk0[s], blk0[s + 1] - 1):
            units.add((int(rng.integers(w.num_q_heads)), int(I)))
    total = int(blk0[-1])
    while len(units) < n:
        units.add((int(rng.integers(w.num_q_heads)), int(rng.integers(total))))
    return sorted(units)

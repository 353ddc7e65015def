"""The attention oracle's tiles evaluated in parallel CPU processes.

Test infrastructure, like the rest of oracle/: only the tests, the smoke
check and the benchmark's CPU-baseline leg use it.  The oracle computes every
(head, q-block) tile independently (osk.osk_units), so a full-size comparison
or a timing can split the tiles over worker processes.  The workers are started
with the 'spawn' method (a process forked after CUDA initialisation hangs) and
read the workload through memory-mapped .npy files written once per workload.
Each worker runs oracle.osk.osk_units on its share of the tiles and returns the
per-tile results: this module only distributes work, it computes nothing.
"""

from __future__ import annotations

import multiprocessing as mp
import os
import shutil
import tempfile

import numpy as np

_DATA: dict = {}
_THREAD_VARS = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")


def _init(paths):
    for key, path in paths.items():
        _DATA[key] = np.load(path, mmap_mode="r")


def _run(job):
    from . import osk
    units, lists, seqlens, num_kv_heads, block_size, tau, q_lens = job
    order = np.load(lists[0], mmap_mode="r")
    count = np.load(lists[1], mmap_mode="r")
    out = []
    for h, I, rows, o, sk, de in osk.osk_units(_DATA["q"], _DATA["k"], _DATA["v"], _DATA["pt"], seqlens,
                                               num_kv_heads, block_size, order, count, tau, units=units,
                                               q_lens=q_lens):
        out.append((h, I, rows.start, rows.stop, o, sk, de))
    return out


class OraclePool:
    """Worker processes holding one workload; run() evaluates tiles of given lists.

    q_bits overrides the workload's Q (prefill after a cached prefix passes the
    query rows only).  Use as a context manager, or call close().
    """

    def __init__(self, w, q_bits=None, workers=None):
        self.w = w
        self.dir = tempfile.mkdtemp(prefix="cosa_oracle_")
        arrays = dict(q=w.q if q_bits is None else q_bits, k=w.k_pages, v=w.v_pages, pt=w.page_table)
        self.paths = {}
        for key, arr in arrays.items():
            self.paths[key] = os.path.join(self.dir, f"{key}.npy")
            np.save(self.paths[key], np.ascontiguousarray(arr))
        self.workers = workers or max(1, min(16, os.cpu_count() or 1))
        saved = {v: os.environ.get(v) for v in _THREAD_VARS}
        for v in _THREAD_VARS:   # one BLAS thread per worker; restored once the workers exist
            os.environ[v] = "1"
        try:
            self.pool = mp.get_context("spawn").Pool(self.workers, initializer=_init, initargs=(self.paths,))
        finally:
            for v, old in saved.items():
                if old is None:
                    os.environ.pop(v, None)
                else:
                    os.environ[v] = old
        self.calls = 0

    def run(self, order, count, tau, units, q_lens=None):
        """{(h, I): (rows, out fp64 [rows, d], skipped bool [k], delta fp64 [k])} for the given units."""
        self.calls += 1
        lists = (os.path.join(self.dir, f"order{self.calls}.npy"), os.path.join(self.dir, f"count{self.calls}.npy"))
        np.save(lists[0], np.ascontiguousarray(order))
        np.save(lists[1], np.ascontiguousarray(count))
        G = self.w.num_q_heads // self.w.num_kv_heads
        units = sorted(set((int(h), int(I)) for h, I in units), key=lambda u: (u[0] // G, u[1], u[0]))
        cost = np.array([max(1, int(count[h, I])) for h, I in units], dtype=np.float64)
        nchunks = min(len(units), self.workers * 4)
        edges = np.searchsorted(np.cumsum(cost), np.linspace(0, cost.sum(), nchunks + 1)[1:-1])
        chunks = [c for c in np.split(np.arange(len(units)), edges) if len(c)]
        seqlens = [int(x) for x in self.w.seqlens]
        jobs = [([units[x] for x in c], lists, seqlens, self.w.num_kv_heads, self.w.block_size, tau, q_lens)
                for c in chunks]
        res = {}
        for part in self.pool.map(_run, jobs):
            for h, I, r0, r1, o, sk, de in part:
                res[(h, I)] = (slice(r0, r1), o, sk, de)
        for path in lists:
            os.remove(path)
        return res

    def close(self):
        if self.pool is not None:
            self.pool.close()
            self.pool.join()
            self.pool = None
        shutil.rmtree(self.dir, ignore_errors=True)

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

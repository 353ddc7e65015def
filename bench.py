"""Benchmark of the CoSA prefill path (KAP proxy + OSK attention) on B200.

One step = one attention layer's prefill through the whole hot path: the
proxy (key pooling, query pooling + exact scores + HRM flags + ordered
selection) and the ordered-skipping attention (page remap in its producer),
on the 128K-token Llama-3.1-8B-shaped layer (32 query heads, 8 KV heads,
head_dim 128, pages of 64 tokens in a shuffled pool, stage-1 budget 5%,
tau = 1e-4).  Inputs are synthetic (seeded), already resident in HBM when
the timed region starts; the 1.5 GiB of inputs per step exceed the 126 MB L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cosa|reference]

Multi-GPU (torchrun): by default one layer is split by kv head across the
ranks (every (head, q-block) tile is independent, so there is no data-path
exchange and the output stays head-sharded); value = the layer's
max-over-ranks time.  --shard layers gives each rank its own layer instead.
The reference arm times the CPU oracle on the same layer: the proxy on all
of it, the attention on a seeded sample of its tiles scaled by visited
blocks to ms per layer (OracleLayer).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill sparse-attn ms/layer @128K; effective TFLOP/s; % TC peak; speedup vs dense"
CONFIG_ID = 3
BUDGET = 0.05
TAU = 1e-4
TAUS = (0.0, 1e-5, 1e-4, 1e-3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sustained=d["bf16_tflops_sustained"],
                    sm_max_mhz=d.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, sm_max_mhz=1965.0, source="fallback")


def tensor_peak(pk, clocks):
    """The dense bf16 peak that matches the clocks sampled in the timed region:
    the burst figure (a cuBLAS GEMM timed alone, at the maximum SM clock) scaled
    by the median SM clock under load over that maximum, capped at 1.  A short
    region runs at the maximum clock, where this is the burst figure itself."""
    mhz = (clocks or {}).get("sm_mhz")
    if not mhz:
        return pk["bf16"], f"{pk['source']} bf16_tflops (burst; no clock samples)"
    ratio = min(1.0, float(mhz) / float(pk["sm_max_mhz"]))
    return pk["bf16"] * ratio, (f"{pk['source']} bf16_tflops (burst, {pk['bf16']:.1f}) x median SM clock "
                                f"{mhz:.0f} / {pk['sm_max_mhz']:.0f} MHz")


def proxy_kernels(w, kmax):
    """The kernels one budget-cut proxy call launches: at head_dim 128 the
    persistent scoring kernel and the register selection (its retry pass always
    launches; kmax <= 128), else the two-stage pool / select kernels."""
    if w.head_dim == 128:
        return ["kpool", "kap_stream", "select_fast", "select_rows"] if kmax <= 128 else \
               ["kpool", "kap_stream", "select_rows"]
    return ["kpool", "qpool", "kap_select"]


def measured_traffic():
    """DRAM bytes per OSK launch from the committed ncu launch list, or None
    when the kernel's sources changed since those counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "osk_traffic_llama8b_128k.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    h = hashlib.sha256()
    for f in d["source_files"]:
        fp = os.path.join(ROOT, f)
        if not os.path.exists(fp):
            return None
        h.update(open(fp, "rb").read())
    if h.hexdigest() != d["source_sha256"]:
        return None
    return d["dram_read_bytes_per_launch"] + d["dram_write_bytes_per_launch"]


def ascending_order(order):
    """The same visited block sets in ascending block order (the -1 padding
    stays last): the visit order of the ablation without the HRM-first order."""
    import torch
    big = torch.iinfo(torch.int32).max
    o = torch.where(order < 0, torch.full_like(order, big), order)
    o = torch.sort(o, dim=-1).values
    return torch.where(o == big, torch.full_like(o, -1), o)


def masked_full_lists(order, count, seqlens, block_size):
    """For the logical-mask ablation: every row's list becomes all its causal
    blocks 0..i in ascending order, with keep = 1 on the blocks the proxy
    selected.  Returns (order_full, count_full, keep, kmax_full)."""
    import torch
    H, N, kmax = order.shape
    dev = order.device
    nqb = [(L + block_size - 1) // block_size for L in seqlens]
    qb_local = torch.cat([torch.arange(n, dtype=torch.int32) for n in nqb]).to(dev)   # [N]
    kmax_full = max(nqb)
    ar = torch.arange(kmax_full, dtype=torch.int32, device=dev)
    full = ar.expand(H, N, kmax_full).clone()
    full[ar.view(1, 1, -1).expand(H, N, -1) > qb_local.view(1, -1, 1).expand(H, -1, kmax_full)] = -1
    count_full = (qb_local + 1).view(1, -1).expand(H, N).contiguous()
    valid = torch.arange(kmax, device=dev).view(1, 1, -1) < count.view(H, N, 1)
    idx = torch.where(valid, order.long(), torch.full_like(order, kmax_full).long())
    keep = torch.zeros((H, N, kmax_full + 1), dtype=torch.uint8, device=dev)
    keep.scatter_(2, idx, valid.to(torch.uint8))
    return full.contiguous(), count_full, keep[:, :, :kmax_full].contiguous(), kmax_full


def rank_seed(cfg, rank, world):
    """Each rank prefills its own independent layer: distinct seeds for N > 1,
    the workload's own seed at N = 1."""
    return None if world == 1 else cfg * 1000 + rank


def head_shard(w, rank, world):
    """Rank `rank`'s share of one layer split by kv head: a contiguous range of
    Hkv / world kv heads (their pages) and the G query heads of each (their
    queries).  Every (head, q-block) tile is independent, so the shards need no
    exchange, and the output stays head-sharded."""
    import dataclasses
    if w.num_kv_heads % world:
        raise ValueError(f"{w.num_kv_heads} kv heads do not split over {world} ranks")
    nkv = w.num_kv_heads // world
    G = w.num_q_heads // w.num_kv_heads
    kv0 = rank * nkv
    return dataclasses.replace(
        w, name=f"{w.name}[kv {kv0}..{kv0 + nkv - 1}]", num_q_heads=nkv * G, num_kv_heads=nkv,
        q=np.ascontiguousarray(w.q[:, kv0 * G:(kv0 + nkv) * G]),
        k_pages=np.ascontiguousarray(w.k_pages[:, kv0:kv0 + nkv]),
        v_pages=np.ascontiguousarray(w.v_pages[:, kv0:kv0 + nkv]),
        meta={**w.meta, "kv_heads": (kv0, kv0 + nkv)})


def max_over_ranks(value, dist=None, device="cuda"):
    """Max of a per-rank duration over all ranks (the job's time)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dense_flops(seqlens, Hq, d):
    return float(sum(4.0 * (L * (L + 1) / 2) * d * Hq for L in seqlens))


def workload_config(w):
    return {"workload": w.name, "seq_len": max(w.seqlens), "batch": w.batch, "num_q_heads": w.num_q_heads,
            "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
            "page_size": w.page_size, "pages": "shuffled pool" if w.meta.get("shuffled_pages") else "contiguous",
            "budget": w.budgets[0], "tau": TAU,
            "l2": "inputs larger than L2 (q 1 GiB + k/v pages 512 MiB per step), no flush"}


class Clocks:
    """nvidia-smi samples (every 50 ms, timestamped) kept only inside the timed region."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(1.5)   # let the sampler come up before the timed region
        except OSError:
            self.proc = None

    def begin(self):
        import datetime
        self.t0 = datetime.datetime.now()

    def end(self):
        import datetime
        self.t1 = datetime.datetime.now()

    def stop(self):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        import datetime
        sm, mx, power, reasons = [], None, [], set()
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f")
                if self.t0 is not None and not (self.t0 <= ts <= self.t1):
                    continue
                sm.append(float(f[2]))
                mx = float(f[3])
                power.append(float(f[4]))
            except ValueError:
                continue
            for n, v in zip(self.REASONS, f[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power)}


# ------------------------------------------------------------------ CPU side

class OracleLayer:
    """The oracle (proxy + OSK) on the bench layer, timed on the host's cores.

    The proxy oracle runs on the whole 128K layer in this process (one thread:
    integer dot products and fp32 sums).  The OSK oracle's tiles are
    independent; a seeded sample of them, drawn from every q-block of the
    layer, runs on worker processes (oracle.parallel.OraclePool, one BLAS
    thread each), and its wall time is scaled to the whole layer by visited
    blocks (the oracle's cost per tile is one fp64 tile product pair per
    visited block)."""

    def __init__(self, workers=None):
        from oracle import kap
        from oracle.parallel import OraclePool
        from synth import make_workload
        self.w = make_workload(CONFIG_ID)
        w = self.w
        t0 = time.perf_counter()
        self.sel = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, BUDGET)
        self.proxy_s = time.perf_counter() - t0
        self.pool = OraclePool(w, workers=workers)
        self.tiles = [(h, I) for h in range(w.num_q_heads) for I in range(self.sel["count"].shape[1])]
        self.visited_all = int(self.sel["count"].sum())

    def sample(self, fraction, seed):
        """(ms per layer estimate, description) from one sample of the OSK tiles."""
        rng = np.random.default_rng(seed)
        n = max(1, int(round(fraction * len(self.tiles))))
        pick = rng.choice(len(self.tiles), size=n, replace=False)
        units = [self.tiles[x] for x in pick]
        visited = int(sum(int(self.sel["count"][h, I]) for h, I in units))
        t0 = time.perf_counter()
        self.pool.run(self.sel["order"], self.sel["count"], TAU, units)
        osk_s = time.perf_counter() - t0
        osk_full = osk_s * self.visited_all / visited
        ms = (self.proxy_s + osk_full) * 1e3
        desc = (f"proxy oracle timed on the whole 128K layer ({self.proxy_s:.1f} s, 1 thread); OSK oracle timed on "
                f"{n} of {len(self.tiles)} (head, q-block) tiles drawn uniformly from the whole layer (seed {seed}): "
                f"{visited} visited blocks in {osk_s:.1f} s on {self.pool.workers} worker processes (1 BLAS thread "
                f"each), scaled by visited blocks to the layer's {self.visited_all} ({osk_full:.1f} s); "
                f"budget {BUDGET}, tau {TAU}")
        return ms, desc

    def close(self):
        self.pool.close()


def run_reference(args, rank, world):
    """The reference arm: the oracle as it stands, on the host's cores (rank 0 only)."""
    if rank != 0:
        return
    layer = OracleLayer()
    try:
        for k in range(args.warmup):
            pass   # the oracle keeps no warm state; warm-up samples are not run, to bound the CPU time
        times, desc = [], ""
        for k in range(args.steps):
            v, desc = layer.sample(args.ref_fraction, seed=1000 + k)
            times.append(v)
    finally:
        layer.close()
    value = statistics.mean(times)
    cb = {"kind": "oracle", "cores": layer.pool.workers, "value": value, "unit": "ms",
          "sample": f"mean over {args.steps} samples; last: {desc}"}
    line = {"metric": METRIC, "value": value, "unit": "ms", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": value, "higher_is_better": False, "scaling": "strong",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": "llama8b_128k", "seq_len": 131072, "budget": BUDGET, "tau": TAU},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU side

def upload(w, device="cuda"):
    """Synthetic workload (bf16 bit patterns in numpy) -> device tensors + Batch."""
    import torch
    import block_sparse_long_14_b200 as cosa

    def bf16(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(device)

    batch = cosa.Batch(w.seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.page_size,
                       w.num_pages, w.max_pages_per_seq, device=device)
    return dict(batch=batch, q=bf16(w.q), k_pages=bf16(w.k_pages), v_pages=bf16(w.v_pages),
                page_table=torch.from_numpy(np.ascontiguousarray(w.page_table)).to(device))


TOP_P = 0.95       # the pages' stage-1 p (Qwen3-8B; Llama's is calibrated per context length)
DELTA = 200.0      # the pages' Llama-3.1-8B delta in tau_s = delta / N


def _timed(fn, stream, reps=2):
    """Device time of fn() on `stream` (ms), after one untimed call."""
    import torch
    fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def pages_rules(cosa, batch, d, nqb_rows, tile_flops, stream):
    """Top-p stage 1 (p = TOP_P) and the length-adaptive tau_s = DELTA / N on the bench layer."""
    ws, kmax = cosa.alloc_workspace(batch, 1.0)     # a Top-p row may keep every candidate
    sel = cosa.proxy_top_p(batch, d["q"], d["k_pages"], d["page_table"], TOP_P, kmax, ws)
    t_proxy = _timed(lambda: cosa.proxy_top_p(batch, d["q"], d["k_pages"], d["page_table"], TOP_P, kmax, ws,
                                              out=sel), stream)
    res = cosa.attn_delta(batch, d["q"], d["k_pages"], d["v_pages"], d["page_table"], sel["order"], sel["count"],
                          kmax, DELTA, ws)
    t_attn = _timed(lambda: cosa.attn_delta(batch, d["q"], d["k_pages"], d["v_pages"], d["page_table"],
                                            sel["order"], sel["count"], kmax, DELTA, ws, out=res), stream)
    cosa.check(ws)
    vis = int(res["visited"].sum().item())
    sk = int(res["skipped"].sum().item())
    return {"p": TOP_P, "delta": DELTA, "ms": t_proxy + t_attn, "proxy_ms": t_proxy, "attn_ms": t_attn,
            "stage1_budget": vis / nqb_rows, "skip_ratio": sk / max(1, vis),
            "stage2_budget": (vis - sk) / nqb_rows,
            "attn_tflops_executed": tile_flops * (2 * vis - sk) / (t_attn * 1e-3) / 1e12}


def cached_prefix(cosa, w, d, budget, stream):
    """The bench layer with its first half as a cached prefix (q_len = kv_len / 2 per sequence)."""
    q_lens = [L - L // 2 for L in w.seqlens]
    rows, tok0 = [], 0
    for L, Lq in zip(w.seqlens, q_lens):
        rows.append(d["q"][tok0 + L - Lq:tok0 + L])
        tok0 += L
    import torch
    q = rows[0] if len(rows) == 1 else torch.cat(rows)
    batch = cosa.Batch(w.seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.page_size,
                       w.num_pages, w.max_pages_per_seq, device="cuda", q_lens=q_lens)
    ws, kmax = cosa.alloc_workspace(batch, budget)
    sel = cosa.proxy(batch, q, d["k_pages"], d["page_table"], budget, kmax, ws)
    t_proxy = _timed(lambda: cosa.proxy(batch, q, d["k_pages"], d["page_table"], budget, kmax, ws, out=sel), stream)
    res = cosa.attn(batch, q, d["k_pages"], d["v_pages"], d["page_table"], sel["order"], sel["count"], kmax, TAU, ws)
    t_attn = _timed(lambda: cosa.attn(batch, q, d["k_pages"], d["v_pages"], d["page_table"], sel["order"],
                                      sel["count"], kmax, TAU, ws, out=res), stream)
    cosa.check(ws)
    return {"q_tokens": sum(q_lens), "kv_tokens": sum(w.seqlens), "budget": budget, "tau": TAU,
            "ms": t_proxy + t_attn, "proxy_ms": t_proxy, "attn_ms": t_attn,
            "skip_ratio": int(res["skipped"].sum().item()) / max(1, int(res["visited"].sum().item()))}


def run_cosa(args, rank, world, local_rank):
    import torch
    import block_sparse_long_14_b200 as cosa
    from synth import make_workload

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist

    if args.shard == "heads":
        w = make_workload(args.config)
        if world > 1:
            w = head_shard(w, rank, world)   # one layer, split by kv head
    else:
        w = make_workload(args.config, seed=rank_seed(args.config, rank, world))
    d = upload(w)
    batch = d["batch"]
    budget = w.budgets[0]
    ws, kmax = cosa.alloc_workspace(batch, budget)
    H, N = w.num_q_heads, batch.total_qblocks
    sel = dict(order=torch.empty((H, N, kmax), dtype=torch.int32, device="cuda"),
               count=torch.empty((H, N), dtype=torch.int32, device="cuda"),
               n_hrm=torch.empty((H, N), dtype=torch.int32, device="cuda"),
               hrm=torch.empty((H, N, kmax), dtype=torch.uint8, device="cuda"))
    res = dict(out=torch.empty_like(d["q"]), visited=torch.empty((H, N), dtype=torch.int32, device="cuda"),
               skipped=torch.empty((H, N), dtype=torch.int32, device="cuda"))
    stream = torch.cuda.current_stream()

    def step(tau=TAU, ev=None):
        if ev is not None:
            ev[0].record(stream)
        cosa.proxy(batch, d["q"], d["k_pages"], d["page_table"], budget, kmax, ws, out=sel)
        if ev is not None:
            ev[1].record(stream)
        cosa.attn(batch, d["q"], d["k_pages"], d["v_pages"], d["page_table"], sel["order"], sel["count"], kmax,
                  tau, ws, out=res)
        if ev is not None:
            ev[2].record(stream)

    clk = Clocks(local_rank)
    clk.start()
    for _ in range(max(3, args.warmup)):
        step()
    cosa.check(ws)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clk.begin()
    start.record(stream)
    for k in range(args.steps):
        step(ev=evs[k])
    stop.record(stream)
    torch.cuda.synchronize()
    clk.end()
    clk.stop()
    if dist is not None:
        dist.barrier()
    cosa.check(ws)
    elapsed = start.elapsed_time(stop)
    t_proxy = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    t_attn = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    elapsed = max_over_ranks(elapsed, dist)
    ms_per_step = elapsed / args.steps
    # ms per layer: the ranks' independent layers run concurrently, or one layer is split
    per_layer = world if args.shard == "layers" else 1
    value = ms_per_step / per_layer

    # ---- work accounting (identical every step)
    visited = int(res["visited"].sum().item())
    skipped = int(res["skipped"].sum().item())
    b, dh = w.block_size, w.head_dim
    tile_flops = 2.0 * b * b * dh
    exec_flops = tile_flops * (visited + (visited - skipped))
    pk = peaks()
    attn_tflops = exec_flops / (t_attn * 1e-3) / 1e12
    q_bytes = w.q.nbytes
    k_bytes = w.k_pages.nbytes
    list_bytes = sum(v.numel() * v.element_size() for v in sel.values())
    proxy_bytes = q_bytes + k_bytes + list_bytes
    proxy_gbs = proxy_bytes / (t_proxy * 1e-3) / 1e9
    dflops = dense_flops(w.seqlens, w.num_q_heads, dh)
    nqb_rows = sum(((L + b - 1) // b) * (((L + b - 1) // b) + 1) // 2 for L in w.seqlens) * w.num_q_heads

    extra = {}
    if rank == 0 and world == 1 and not args.quick:
        # tau sweep (device-timed, same inputs)
        sweep = {}
        for tau in TAUS:
            for _ in range(2):
                step(tau)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            ts = []
            for _ in range(3):
                step(tau, ev=e)
                torch.cuda.synchronize()
                ts.append((e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2])))
            vis = int(res["visited"].sum().item())
            sk = int(res["skipped"].sum().item())
            ta = statistics.mean(x[1] for x in ts)
            tp = statistics.mean(x[0] for x in ts)
            sweep[str(tau)] = {"ms": tp + ta, "proxy_ms": tp, "attn_ms": ta, "skip_ratio": sk / vis,
                               "attn_tflops_executed": tile_flops * (2 * vis - sk) / (ta * 1e-3) / 1e12,
                               "stage2_budget": (vis - sk) / nqb_rows}
        extra["tau_sweep"] = sweep
        cosa.check(ws)
        # visit-order ablation: the proxy's lists (HRM first, then by score) against the
        # same block sets in ascending block order, at fixed tau
        step(TAU)
        torch.cuda.synchronize()
        orders = {"hrm_first": sel["order"].clone(), "ascending": ascending_order(sel["order"])}
        abl = {}
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for tau in (1e-4, 1e-3):
            for name, ordr in orders.items():
                cosa.attn(batch, d["q"], d["k_pages"], d["v_pages"], d["page_table"], ordr, sel["count"], kmax,
                          tau, ws, out=res)
                e0.record(stream)
                cosa.attn(batch, d["q"], d["k_pages"], d["v_pages"], d["page_table"], ordr, sel["count"], kmax,
                          tau, ws, out=res)
                e1.record(stream)
                torch.cuda.synchronize()
                vis = int(res["visited"].sum().item())
                sk = int(res["skipped"].sum().item())
                abl[f"{name}@{tau}"] = {"attn_ms": e0.elapsed_time(e1), "skip_ratio": sk / vis}
        cosa.check(ws)
        # logical-mask execution of the ascending run: every causal block is walked, the
        # unselected ones passed over with a mask check (physical jumping vs a mask loop)
        o_full, c_full, keep, kmax_full = masked_full_lists(sel["order"], sel["count"], w.seqlens, w.block_size)
        ws_m, _ = cosa.alloc_workspace(batch, 1.0)
        for tau in (1e-4, 1e-3):
            cosa.attn_masked(batch, d["q"], d["k_pages"], d["v_pages"], d["page_table"], o_full, c_full, kmax_full,
                             keep, tau, ws_m, out=res)
            e0.record(stream)
            cosa.attn_masked(batch, d["q"], d["k_pages"], d["v_pages"], d["page_table"], o_full, c_full, kmax_full,
                             keep, tau, ws_m, out=res)
            e1.record(stream)
            torch.cuda.synchronize()
            vis = int(res["visited"].sum().item())
            sk = int(res["skipped"].sum().item())
            abl[f"mask_loop@{tau}"] = {"attn_ms": e0.elapsed_time(e1), "skip_ratio": sk / vis,
                                       "entries_walked": int(c_full.sum().item())}
        cosa.check(ws_m)
        del o_full, c_full, keep, ws_m
        extra["order_ablation"] = abl
        # dense reference on the same B200: our OSK at budget 100% / tau 0, and torch SDPA (flash)
        ws_d, kmax_d = cosa.alloc_workspace(batch, 1.0)
        sel_d = cosa.proxy(batch, d["q"], d["k_pages"], d["page_table"], 1.0, kmax_d, ws_d)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cosa.attn(batch, d["q"], d["k_pages"], d["v_pages"], d["page_table"], sel_d["order"], sel_d["count"],
                  kmax_d, 0.0, ws_d, out=res)
        e0.record(stream)
        cosa.attn(batch, d["q"], d["k_pages"], d["v_pages"], d["page_table"], sel_d["order"], sel_d["count"],
                  kmax_d, 0.0, ws_d, out=res)
        e1.record(stream)
        torch.cuda.synchronize()
        cosa.check(ws_d)
        dense_osk_ms = e0.elapsed_time(e1)
        del sel_d, ws_d
        sdpa_ms = None
        try:
            L = w.seqlens[0]
            G = w.num_q_heads // w.num_kv_heads
            qd = d["q"].view(L, w.num_q_heads, dh).transpose(0, 1).unsqueeze(0)
            kd = torch.randn((1, w.num_kv_heads, L, dh), dtype=torch.bfloat16, device="cuda")
            vd = torch.randn_like(kd)
            sdpa = torch.nn.functional.scaled_dot_product_attention
            sdpa(qd, kd, vd, is_causal=True, enable_gqa=True)
            e0.record(stream)
            sdpa(qd, kd, vd, is_causal=True, enable_gqa=True)
            e1.record(stream)
            torch.cuda.synchronize()
            sdpa_ms = e0.elapsed_time(e1)
            del kd, vd
        except Exception as exc:  # library reference only
            extra["sdpa_error"] = str(exc)[:200]
        extra["dense"] = {"osk_full_budget_tau0_ms": dense_osk_ms, "torch_sdpa_flash_ms": sdpa_ms,
                          "dense_tflop": dflops / 1e12}
        extra["speedup_vs_dense"] = {"vs_osk_dense": dense_osk_ms / ms_per_step,
                                     "vs_torch_sdpa": (sdpa_ms / ms_per_step) if sdpa_ms else None}

    # ---- end to end through the public API: pinned host inputs in, results out
    e2e = None
    if not args.quick:
        h_q = torch.empty(d["q"].shape, dtype=torch.bfloat16, pin_memory=True)
        h_k = torch.empty(d["k_pages"].shape, dtype=torch.bfloat16, pin_memory=True)
        h_v = torch.empty(d["v_pages"].shape, dtype=torch.bfloat16, pin_memory=True)
        h_t = torch.empty(d["page_table"].shape, dtype=torch.int32, pin_memory=True)
        h_q.copy_(d["q"])
        h_k.copy_(d["k_pages"])
        h_v.copy_(d["v_pages"])
        h_t.copy_(d["page_table"])
        h_out = torch.empty(res["out"].shape, dtype=torch.bfloat16, pin_memory=True)
        h_vis = torch.empty(res["visited"].shape, dtype=torch.int32, pin_memory=True)
        h_skp = torch.empty_like(h_vis, pin_memory=True)

        def e2e_step():
            d["q"].copy_(h_q, non_blocking=True)
            d["k_pages"].copy_(h_k, non_blocking=True)
            d["v_pages"].copy_(h_v, non_blocking=True)
            d["page_table"].copy_(h_t, non_blocking=True)
            step()
            h_out.copy_(res["out"], non_blocking=True)
            h_vis.copy_(res["visited"], non_blocking=True)
            h_skp.copy_(res["skipped"], non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        k2 = max(2, min(args.steps, 5))
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(k2):
            e2e_step()
        stop.record(stream)
        torch.cuda.synchronize()
        el = start.elapsed_time(stop)
        el = max_over_ranks(el, dist)
        cosa.check(ws)
        h2d = h_q.nbytes + h_k.nbytes + h_v.nbytes + h_t.nbytes
        d2h = h_out.nbytes + h_vis.nbytes + h_skp.nbytes
        e2e = {"value": el / k2 / per_layer, "unit": "ms", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": k2}

    if rank == 0 and world == 1 and not args.quick:
        # Informational legs, run after every number the headline line needs: the
        # pages' own stage rules on the same layer (Top-p stage 1, tau_s = delta / N),
        # and the layer as prefill after a cached prefix (its first half has keys and
        # values but no queries).
        try:
            extra["pages_rules"] = pages_rules(cosa, batch, d, nqb_rows, tile_flops, stream)
        except Exception as exc:
            extra["pages_rules"] = {"error": str(exc)[:200]}
        try:
            extra["cached_prefix"] = cached_prefix(cosa, w, d, budget, stream)
        except Exception as exc:
            extra["cached_prefix"] = {"error": str(exc)[:200]}

    if rank != 0:
        return
    clocks = clk.summary()
    tc_peak, tc_peak_source = tensor_peak(pk, clocks)
    line = {
        "metric": METRIC, "value": value, "unit": "ms", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": False,
        "scaling": "weak" if args.shard == "layers" else "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "cosa",
        "config": {**workload_config(w), "parallelism": "single" if world == 1 else
                   (f"independent layers x{world}" if args.shard == "layers" else f"kv-head shards x{world}")},
        "breakdown_ms": {"proxy": t_proxy, "attn": t_attn},
        "effective_tflops": world * dflops / (ms_per_step * 1e-3) / 1e12,   # all ranks' work
        "attn_executed_tflops": attn_tflops,
        "pct_tc_peak": attn_tflops / tc_peak,
        "proxy_gbs": proxy_gbs,
        "pct_hbm_proxy": proxy_gbs / pk["hbm_gbs"],
        "realized_budget": {"stage1": visited / nqb_rows, "stage2": (visited - skipped) / nqb_rows,
                            "skip_ratio": skipped / visited},
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": attn_tflops / tc_peak,
                     "traffic": measured_traffic() if CONFIG_ID == args.config else None,
                     "kernel": "osk_kernel<128,128>",
                     "peak_source": tc_peak_source,
                     "algorithmic": f"{exec_flops:.4e} FLOP per launch = 2*128*128*128 * (visited + kept)"},
        "proxy_roofline": {"bound": "hbm", "achieved": proxy_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                           "frac": proxy_gbs / pk["hbm_gbs"], "algorithmic_bytes": proxy_bytes,
                           "kernels": " + ".join(proxy_kernels(w, kmax))},
        "clocks": clocks,
        "gpu_launches": (len(proxy_kernels(w, kmax)) + 1) * args.steps,   # the proxy's kernels and osk per step
        "e2e": e2e,
        **extra,
    }
    if world == 1 and not args.no_cpu_baseline:
        layer = OracleLayer()
        try:
            v, desc = layer.sample(args.ref_fraction, seed=CONFIG_ID)
        finally:
            layer.close()
        line["cpu_baseline"] = {"value": v, "unit": "ms", "cores": layer.pool.workers, "kind": "oracle",
                                "sample": desc}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cosa", choices=["cosa", "reference"])
    ap.add_argument("--config", type=int, default=CONFIG_ID)
    ap.add_argument("--quick", action="store_true", help="skip the tau sweep, dense reference and e2e legs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-fraction", type=float, default=0.03,
                    help="share of the layer's (head, q-block) tiles the oracle's OSK leg times per sample")
    ap.add_argument("--shard", default="heads", choices=["layers", "heads"],
                    help="N > 1: one layer split by kv head across the ranks (default; strong scaling, "
                         "no exchange) or each rank its own layer (weak scaling)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_cosa(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

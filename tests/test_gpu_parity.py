"""GPU parity: libcosa (through its C ABI) vs the CPU oracle, element by element.

Small packed batches that finish in seconds on the oracle yet span several
tiles, ragged tails, partial pages, several page sizes, head_dim 64/128,
block size 64/128 and GQA groups 1/4/8.
"""

import functools

import numpy as np
import pytest
import torch

import block_sparse_long_14_b200 as cosa
from oracle import dense, kap, osk
from synth import make_custom, make_workload
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": lambda: make_workload(1),
    "ragged_b128_p64": lambda: make_custom([1000, 300, 2100, 129], 8, 2, 128, 128, 64, structure="llama", seed=21),
    "ragged_b128_p16_g1": lambda: make_custom([700, 1500], 4, 4, 128, 128, 16, structure="llama", seed=22),
    "d64_b128_p32": lambda: make_custom([1200, 513], 4, 2, 64, 128, 32, structure="llama", seed=23),
    "b64_g8": lambda: make_custom([900, 200], 16, 2, 128, 64, 64, structure="llama", seed=24),
    "short_seqs": lambda: make_custom([50, 128, 1, 129], 4, 1, 128, 128, 64, structure="random", seed=25),
    "qwen_mix": lambda: make_custom([1500], 32, 8, 128, 128, 64, structure="qwen", seed=26),
}


@functools.lru_cache(maxsize=None)
def workload(name):
    return CASES[name]()


@functools.lru_cache(maxsize=None)
def oracle_proxy(name, budget):
    w = workload(name)
    return kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, budget)


@functools.lru_cache(maxsize=None)
def oracle_attn(name, budget, tau):
    w = workload(name)
    r = oracle_proxy(name, budget)
    return osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size,
                   r["order"], r["count"], tau)


@functools.lru_cache(maxsize=None)
def device(name):
    return gu.upload(workload(name))


@pytest.mark.parametrize("budget", [0.25, 1.0, 0.05])
@pytest.mark.parametrize("name", list(CASES))
def test_proxy_bit_exact(name, budget):
    got, kmax, _ = gu.run_proxy(device(name), budget)
    ref = oracle_proxy(name, budget)
    assert kmax == ref["kmax"]
    gu.assert_proxy_equal(got, ref)


@pytest.mark.parametrize("name", list(CASES))
def test_remap_bit_exact(name):
    w, d = workload(name), device(name)
    ws, kmax = cosa.alloc_workspace(d["batch"], 0.25)
    sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], 0.25, kmax, ws)
    pages = cosa.remap(d["batch"], d["page_table"], sel["order"], sel["count"], kmax)
    cosa.check(ws)
    ref = oracle_proxy(name, 0.25)
    expect = kap.remap(ref["order"], ref["count"], w.page_table, w.seqlens, w.block_size, w.page_size)
    assert np.array_equal(pages.cpu().numpy(), expect)


@pytest.mark.parametrize("budget,tau", [(0.25, 1e-4), (0.25, 0.0), (1.0, 1e-2), (0.25, 1e-2)])
@pytest.mark.parametrize("name", list(CASES))
def test_attn_matches_oracle(name, budget, tau):
    w, d = workload(name), device(name)
    ws, kmax = cosa.alloc_workspace(d["batch"], budget)
    sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], budget, kmax, ws)
    res = gu.run_attn(d, sel, kmax, tau, ws)
    ref = oracle_attn(name, budget, tau)
    stats = gu.compare_attn(res, ref, w, tau, gu.all_units(w))
    if tau == 0.0:
        assert int(res["skipped"].sum()) == 0
    print(name, budget, tau, stats)


@pytest.mark.parametrize("name", ["tiny", "ragged_b128_p64", "b64_g8"])
def test_full_budget_no_skip_equals_dense(name):
    """Budget 100% and tau = 0: OSK is dense causal attention (fp64 brute force)."""
    w, d = workload(name), device(name)
    ws, kmax = cosa.alloc_workspace(d["batch"], 1.0)
    sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], 1.0, kmax, ws)
    res = gu.run_attn(d, sel, kmax, 0.0, ws)
    ref = dense.dense_causal(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads)
    err = np.abs(res["out"].float().cpu().numpy() - ref)
    assert err.max() <= gu.MAX_ABS and err.mean() <= gu.MEAN_ABS


def test_order_invariance_on_gpu():
    """tau = 0: a random permutation of every visit list changes only rounding."""
    name = "ragged_b128_p64"
    d = device(name)
    ws, kmax = cosa.alloc_workspace(d["batch"], 0.25)
    sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], 0.25, kmax, ws)
    a = gu.run_attn(d, sel, kmax, 0.0, ws)["out"].float()
    order = sel["order"].clone()
    cnt = sel["count"].cpu().numpy()
    o = order.cpu().numpy()
    rng = np.random.default_rng(3)
    for h in range(o.shape[0]):
        for I in range(o.shape[1]):
            o[h, I, :cnt[h, I]] = rng.permutation(o[h, I, :cnt[h, I]])
    perm = torch.from_numpy(o).cuda()
    b = gu.run_attn(d, dict(order=perm, count=sel["count"]), kmax, 0.0, ws)["out"].float()
    assert (a - b).abs().max().item() <= gu.MAX_ABS
    assert (a - b).abs().mean().item() <= gu.MEAN_ABS


def ascending_rows(order, count):
    """Each row's visited blocks in ascending block order (the -1 padding stays last)."""
    o = order.copy()
    for h in range(o.shape[0]):
        for I in range(o.shape[1]):
            o[h, I, :count[h, I]] = np.sort(o[h, I, :count[h, I]])
    return o


@pytest.mark.parametrize("name,tau", [("ragged_b128_p64", 1e-3), ("qwen_mix", 1e-2)])
def test_attn_ascending_order_matches_oracle(name, tau):
    """Visit-order ablation: the same block sets visited in ascending block order
    (no HRM-first order) match the oracle run on that order, skip sets included."""
    budget = 0.25
    w, d = workload(name), device(name)
    ws, kmax = cosa.alloc_workspace(d["batch"], budget)
    sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], budget, kmax, ws)
    cnt = sel["count"].cpu().numpy()
    asc = torch.from_numpy(ascending_rows(sel["order"].cpu().numpy(), cnt)).cuda()
    res = gu.run_attn(d, dict(order=asc, count=sel["count"]), kmax, tau, ws)
    r = oracle_proxy(name, budget)
    ref = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size,
                  ascending_rows(r["order"], r["count"]), r["count"], tau)
    stats = gu.compare_attn(res, ref, w, tau, gu.all_units(w))
    print(name, tau, stats)


@pytest.mark.parametrize("name,delta", [("ragged_b128_p64", 20.0), ("short_seqs", 2.0), ("ragged_b128_p64", -1.0)])
def test_attn_delta_matches_oracle_per_sequence(name, delta):
    """tau_s = delta / L_s per sequence (the pages' length-adaptive threshold),
    against the oracle run sequence by sequence with that sequence's tau."""
    budget = 0.25
    w, d = workload(name), device(name)
    ws, kmax = cosa.alloc_workspace(d["batch"], budget)
    sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], budget, kmax, ws)
    res = cosa.attn_delta(d["batch"], d["q"], d["k_pages"], d["v_pages"], d["page_table"], sel["order"],
                          sel["count"], kmax, delta, ws, skipbits=True)
    cosa.check(ws)
    r = oracle_proxy(name, budget)
    b = w.block_size
    nqb = [(L + b - 1) // b for L in w.seqlens]
    qb0 = np.concatenate([[0], np.cumsum(nqb)])
    for s_i, L in enumerate(w.seqlens):
        tau = 0.0 if delta == -1.0 else delta / L
        units = [(h, I) for h in range(w.num_q_heads) for I in range(qb0[s_i], qb0[s_i + 1])]
        ref = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size,
                      r["order"], r["count"], tau, units=units)
        stats = gu.compare_attn(res, ref, w, tau, units)
        print(name, delta, s_i, L, tau, stats)
    if delta == -1.0:
        assert int(res["skipped"].sum()) == 0


@pytest.mark.parametrize("name,tau", [("ragged_b128_p64", 1e-3), ("qwen_mix", 1e-2), ("short_seqs", 1e-4)])
def test_mask_loop_equals_physical_jump(name, tau):
    """Logical-mask execution (every causal block walked, the unselected ones
    passed over) computes exactly what the jump over the same blocks in
    ascending order computes: same output bits, same counts."""
    import bench
    budget = 0.25
    w, d = workload(name), device(name)
    ws, kmax = cosa.alloc_workspace(d["batch"], budget)
    sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], budget, kmax, ws)
    asc = bench.ascending_order(sel["order"])
    jump = cosa.attn(d["batch"], d["q"], d["k_pages"], d["v_pages"], d["page_table"], asc, sel["count"], kmax, tau,
                     ws)
    cosa.check(ws)
    o_full, c_full, keep, kmax_full = bench.masked_full_lists(sel["order"], sel["count"], w.seqlens, w.block_size)
    ws_m, _ = cosa.alloc_workspace(d["batch"], 1.0)
    mask = cosa.attn_masked(d["batch"], d["q"], d["k_pages"], d["v_pages"], d["page_table"], o_full, c_full,
                            kmax_full, keep, tau, ws_m, skipbits=True)
    cosa.check(ws_m)
    assert torch.equal(mask["visited"], sel["count"])
    assert torch.equal(mask["skipped"], jump["skipped"])
    assert torch.equal(mask["out"], jump["out"])
    # skip bits sit at list entries: exactly the kept entries can carry one
    assert int((mask["skipbits"].int() * (1 - keep.int())).sum()) == 0
    assert int(mask["skipbits"].int().sum()) == int(jump["skipped"].sum())


@pytest.mark.parametrize("name", ["ragged_b128_p64", "ragged_b128_p16_g1", "d64_b128_p32", "b64_g8"])
def test_nhd_pages_give_identical_results(name):
    """The same pools stored [P, b_p, Hkv, d] (NHD) instead of [P, Hkv, b_p, d]:
    identical lists, HRM flags, outputs and skip decisions."""
    budget, tau = 0.25, 1e-3
    w, d = workload(name), device(name)
    ws, kmax = cosa.alloc_workspace(d["batch"], budget)
    sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], budget, kmax, ws)
    sel = {k: v.clone() for k, v in sel.items()}
    res = gu.run_attn(d, sel, kmax, tau, ws)
    kn = d["k_pages"].permute(0, 2, 1, 3).contiguous()
    vn = d["v_pages"].permute(0, 2, 1, 3).contiguous()
    bn = cosa.Batch(w.seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.page_size, w.num_pages,
                    w.max_pages_per_seq, page_layout=cosa.PAGES_NHD)
    sel_n = cosa.proxy(bn, d["q"], kn, d["page_table"], budget, kmax, ws)
    cosa.check(ws)
    for k in sel:
        assert torch.equal(sel_n[k], sel[k]), k
    res_n = cosa.attn(bn, d["q"], kn, vn, d["page_table"], sel_n["order"], sel_n["count"], kmax, tau, ws,
                      skipbits=True)
    cosa.check(ws)
    for k in ("out", "visited", "skipped", "skipbits"):
        assert torch.equal(res_n[k], res[k]), k


def test_repeated_calls_are_deterministic():
    d = device("qwen_mix")
    ws, kmax = cosa.alloc_workspace(d["batch"], 0.25)
    outs = []
    for _ in range(3):
        sel = cosa.proxy(d["batch"], d["q"], d["k_pages"], d["page_table"], 0.25, kmax, ws)
        r = gu.run_attn(d, sel, kmax, 1e-4, ws)
        outs.append((sel["order"].clone(), r["out"].clone(), r["skipped"].clone()))
    for o in outs[1:]:
        assert torch.equal(o[0], outs[0][0]) and torch.equal(o[1], outs[0][1]) and torch.equal(o[2], outs[0][2])


# Prefill after a cached prefix: queries are each sequence's last q_len tokens.
# Prefixes on and off the block grid, two whole sub-rows absent, single-query
# sequences, and the d = 64 proxy path.
PREFIX_CASES = {
    "ragged_b128_p64": [1000 - 384, 300, 2100 - 1000, 1],
    "b64_g8": [900 - 100, 200 - 163],
    "short_seqs": [50, 1, 1, 64],
    "d64_b128_p32": [1200 - 256, 513 - 200],
}


@functools.lru_cache(maxsize=None)
def oracle_prefix(name, budget):
    w, q_lens = workload(name), PREFIX_CASES[name]
    return kap.kap_proxy(gu.prefix_q(w, q_lens), w.k_pages, w.page_table, w.seqlens, w.num_kv_heads,
                         w.block_size, budget, q_lens=q_lens)


@pytest.mark.parametrize("budget,tau", [(0.25, 1e-3), (1.0, 0.0)])
@pytest.mark.parametrize("name", list(PREFIX_CASES))
def test_prefix_prefill_matches_oracle(name, budget, tau):
    """Proxy lists (workspace and allocation-free paths) and remap bit-exact,
    attention within tolerance, for prefill after a cached prefix."""
    w, q_lens = workload(name), PREFIX_CASES[name]
    d = gu.upload(w, q_lens=q_lens)
    got, kmax, ws = gu.run_proxy(d, budget)
    ref = oracle_prefix(name, budget)
    assert kmax == ref["kmax"]
    gu.assert_proxy_equal(got, ref)
    na = cosa.proxy_noalloc(d["batch"], d["q"], d["k_pages"], d["page_table"], budget, kmax)
    torch.cuda.synchronize()
    gu.assert_proxy_equal({k: v.cpu().numpy() for k, v in na.items()}, ref)
    sel = {k: torch.from_numpy(v).cuda() for k, v in got.items()}
    pages = cosa.remap(d["batch"], d["page_table"], sel["order"], sel["count"], kmax)
    expect = kap.remap(ref["order"], ref["count"], w.page_table, w.seqlens, w.block_size, w.page_size,
                       q_lens=q_lens)
    assert np.array_equal(pages.cpu().numpy(), expect)
    res = gu.run_attn(d, sel, kmax, tau, ws)
    qp = gu.prefix_q(w, q_lens)
    o = osk.osk(qp, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, ref["order"],
                ref["count"], tau, q_lens=q_lens)
    units = [(h, I) for h in range(w.num_q_heads) for I in range(ref["count"].shape[1])]
    stats = gu.compare_attn(res, o, w, tau, units, q_lens=q_lens)
    if budget == 1.0 and tau == 0.0:
        dn = dense.dense_causal(qp, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, q_lens=q_lens)
        err = np.abs(res["out"].float().cpu().numpy() - dn)
        assert err.max() <= gu.MAX_ABS and err.mean() <= gu.MEAN_ABS
    print(name, budget, tau, stats)


TOP_P_EPS = 1e-5   # a cut whose oracle share lies within this of p may fall on either side


@pytest.mark.parametrize("p", [0.5, 0.9, 0.95, 1.0])
@pytest.mark.parametrize("name", ["tiny", "ragged_b128_p64", "qwen_mix", "d64_b128_p32", "b64_g8"])
def test_proxy_top_p_matches_oracle(name, p):
    """The Top-p cut: each row's count within the oracle's window around p,
    and its entries the leading entries of the full flag-grouped order."""
    w, d = workload(name), device(name)
    ws, kmax = cosa.alloc_workspace(d["batch"], 1.0)
    sel = cosa.proxy_top_p(d["batch"], d["q"], d["k_pages"], d["page_table"], p, kmax, ws)
    cosa.check(ws)
    got = {k: v.cpu().numpy() for k, v in sel.items()}
    ref = kap.kap_proxy_top_p(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, p,
                              eps=TOP_P_EPS)
    full = oracle_proxy(name, 1.0)
    assert kmax == full["kmax"] == ref["kmax"]
    cnt = got["count"]
    assert np.all(ref["count_lo"] <= cnt) and np.all(cnt <= ref["count_hi"])
    Hq, NQB = cnt.shape
    for h in range(Hq):
        for I in range(NQB):
            k = int(cnt[h, I])
            assert 1 <= k <= full["count"][h, I]
            assert got["order"][h, I, :k].tolist() == full["order"][h, I, :k].tolist()
            assert np.all(got["order"][h, I, k:] == -1)
            assert got["hrm"][h, I, :k].tolist() == full["hrm"][h, I, :k].tolist()
            assert not got["hrm"][h, I, k:].any()
            assert got["n_hrm"][h, I] == int(full["hrm"][h, I, :k].sum())
    if p == 1.0:
        assert np.array_equal(cnt, full["count"])
    print(name, p, "exact", float((cnt == ref["count"]).mean()), "mean k", float(cnt.mean()))


@pytest.mark.parametrize("name,p,tau", [("ragged_b128_p64", 0.95, 1e-3), ("qwen_mix", 0.9, 1e-4)])
def test_attn_on_top_p_lists_matches_oracle(name, p, tau):
    """The OSK over the (long) lists of the Top-p rule, the oracle's lists given to both sides."""
    w, d = workload(name), device(name)
    ref = kap.kap_proxy_top_p(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, p)
    ws, _ = cosa.alloc_workspace(d["batch"], 1.0)
    sel = {"order": torch.from_numpy(ref["order"]).cuda(), "count": torch.from_numpy(ref["count"]).cuda()}
    res = gu.run_attn(d, sel, ref["kmax"], tau, ws)
    o = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, ref["order"],
                ref["count"], tau)
    print(name, p, tau, gu.compare_attn(res, o, w, tau, gu.all_units(w)))


def _zero_blocks_workload():
    """Random Q/K/V (700 tokens, b = 128) with key block 1 all zero (scale 0),
    one all-zero 16-row query sub-row in q-block 2 and q-block 4 all zero
    (every score 0: ties broken by the lowest block index)."""
    from synth import from_arrays
    rng = np.random.default_rng(31)
    L = 700
    q = rng.standard_normal((L, 4, 128)).astype(np.float32)
    k = rng.standard_normal((L, 2, 128)).astype(np.float32)
    v = rng.standard_normal((L, 2, 128)).astype(np.float32)
    k[128:256] = 0.0
    q[288:304] = 0.0
    q[512:640] = 0.0
    return from_arrays([q], [k], [v], 128, 64, shuffle=True, seed=31)


@pytest.mark.parametrize("budget,tau", [(0.25, 1e-3), (0.001, 1e-4)])
def test_zero_blocks_and_single_entry_lists(budget, tau):
    """Edge cases: an all-zero key block and zero query vectors (quantised to
    zero with scale 0), and budget 0.1 %, where every list holds one entry (kmax = 1)."""
    w = _zero_blocks_workload()
    d = gu.upload(w)
    got, kmax, ws = gu.run_proxy(d, budget)
    ref = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, budget)
    assert kmax == ref["kmax"]
    if budget == 0.001:
        assert kmax == 1
    gu.assert_proxy_equal(got, ref)
    sel = {k: torch.from_numpy(v).cuda() for k, v in got.items()}
    res = gu.run_attn(d, sel, kmax, tau, ws)
    o = osk.osk(w.q, w.k_pages, w.v_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, ref["order"],
                ref["count"], tau)
    print(budget, tau, gu.compare_attn(res, o, w, tau, gu.all_units(w)))


def _sample_defeating_workload():
    """One 64K-token sequence (b = 128: rows of up to 512 candidates), two kv
    heads, one query head each, with every query token equal.  Each key block
    is a constant vector s_j u, so block j's proxy score is proportional to
    s_j.  For the last q-block (n = 512) the 64 threshold samples of the
    register selection sit at blocks 8e.  Kv head 0 gives those 64 blocks the
    highest scores: at a 5 % budget (k = 26) no sample rank tried (the 6th,
    10th and 16th smallest) has k keys at or below it (nor within the
    threshold's lowest score bit of it).  Kv head 1 gives them
    the lowest scores: every sample has more than the 256 keys the kept buffer
    holds below it.  Both rows must finish in the shared-memory selection."""
    from synth import from_arrays
    rng = np.random.default_rng(41)
    nb, b, d = 512, 128, 128
    L = nb * b
    u = np.ones(d, dtype=np.float32) / np.sqrt(d)
    on = np.zeros(nb, dtype=bool)
    on[::8] = True
    hi = 2.0 + 6.0 * rng.random(nb)    # few equal bf16 values among the 64 sampled blocks
    lo = -1.0 - 6.0 * rng.random(nb)
    s = np.stack([np.where(on, hi, lo), np.where(on, -hi, -lo)], axis=1)   # [nb, kv head]
    k = np.repeat(s, b, axis=0)[:, :, None] * u[None, None, :]
    q = np.broadcast_to(u, (L, 2, d)).astype(np.float32)
    v = rng.standard_normal((L, 2, d)).astype(np.float32)
    return from_arrays([q], [k.astype(np.float32)], [v], b, 128, shuffle=True, seed=41)


def test_selection_rows_the_register_path_leaves():
    """Rows whose sampled threshold fails (too few keys below every sample
    tried, or more than the kept buffer holds) are finished by the
    shared-memory selection through the retry list: the lists are bit-exact
    and both constructed rows are on the list."""
    w = _sample_defeating_workload()
    d = gu.upload(w)
    got, kmax, ws = gu.run_proxy(d, 0.05)
    ref = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, 0.05)
    assert kmax == ref["kmax"] == 26
    gu.assert_proxy_equal(got, ref)
    # the retry list is the workspace's last region: a count, then one entry per row
    rows = w.num_q_heads * d["batch"].total_qblocks
    region = (4 * (1 + rows) + 255) // 256 * 256
    lst = ws[ws.numel() - region:].view(torch.int32).cpu().numpy()
    listed = set(lst[1:1 + lst[0]].tolist())
    # rows are numbered (q-blocks from the last) * heads + head: the last q-block's are 0 and 1
    assert {0, 1} <= listed, (lst[0], sorted(listed)[:8])
    assert all(0 <= r < rows for r in listed)

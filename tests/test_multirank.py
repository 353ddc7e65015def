"""The benchmark's multi-GPU host logic on CPU with 2 gloo ranks.

With N GPUs every rank prefills its own independent layer (the default), or
the ranks split one layer by kv head (--shard heads); either way there is no
data-path collective, and the job time is the max over ranks.  Checked here
without a GPU: distinct per-rank workloads, an exact partition of the heads,
shard lists equal to the full layer's, and the max-over-ranks reduction.
"""

import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    from synth import make_custom
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        seed = bench.rank_seed(3, rank, world)
        w = make_custom([300], 4, 2, 64, 64, 32, structure="llama", seed=seed)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, dist, device="cpu")
        digest = int(np.asarray(w.q[:64], dtype=np.int64).sum())
        q.put((rank, seed, t, digest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_run_independent_layers_and_take_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got[0][1] != got[1][1]                 # distinct seeds
    assert got[0][3] != got[1][3]                 # distinct inputs
    assert got[0][2] == got[1][2] == 15.0         # job time = max over ranks


def test_single_rank_uses_the_workload_seed():
    import bench
    assert bench.rank_seed(3, 0, 1) is None
    assert bench.max_over_ranks(7.5) == 7.5


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    from synth import make_custom
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        full = make_custom([300, 130], 8, 4, 64, 64, 32, structure="llama", seed=7)   # same layer on every rank
        w = bench.head_shard(full, rank, world)
        t = bench.max_over_ranks(3.0 * (rank + 1), dist, device="cpu")
        q.put((rank, w.meta["kv_heads"], w.num_q_heads, w.num_kv_heads, w.q, w.k_pages, w.v_pages, t))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_one_layer_by_kv_head():
    """--shard heads: the ranks' shards partition the layer's heads exactly,
    with no data exchanged, and the job time is the max over ranks."""
    from synth import make_custom
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=120) for _ in range(2)), key=lambda x: x[0])
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    full = make_custom([300, 130], 8, 4, 64, 64, 32, structure="llama", seed=7)
    assert [g[1] for g in got] == [(0, 2), (2, 4)]
    assert all(g[2] == 4 and g[3] == 2 for g in got)
    assert np.array_equal(np.concatenate([g[4] for g in got], axis=1), full.q)
    assert np.array_equal(np.concatenate([g[5] for g in got], axis=1), full.k_pages)
    assert np.array_equal(np.concatenate([g[6] for g in got], axis=1), full.v_pages)
    assert got[0][7] == got[1][7] == 6.0


def test_head_shards_give_the_full_layers_lists():
    """Tiles are independent: the oracle's lists for a kv-head shard are the
    full layer's lists for those query heads."""
    import bench
    from oracle import kap
    from synth import make_custom
    full = make_custom([300, 130], 8, 4, 64, 64, 32, structure="llama", seed=7)
    ref = kap.kap_proxy(full.q, full.k_pages, full.page_table, full.seqlens, 4, 64, 0.3)
    for rank in range(4):
        w = bench.head_shard(full, rank, 4)
        r = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, 64, 0.3)
        h0, h1 = 2 * rank, 2 * rank + 2
        for key in ("order", "count", "n_hrm", "hrm"):
            assert np.array_equal(r[key], ref[key][h0:h1]), key
    try:
        bench.head_shard(full, 0, 3)
        raise AssertionError("4 kv heads split over 3 ranks")
    except ValueError:
        pass

"""The benchmark's multi-GPU host logic on CPU with 2 gloo ranks.

With N GPUs every rank prefills its own independent layer (no data-path
collective); the job time is the max over ranks.  Checked here without a GPU:
distinct per-rank workloads and the max-over-ranks reduction.
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

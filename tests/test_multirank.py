"""bench.py's multi-rank plumbing on CPU ranks (gloo, world size 2): rank
setup, barrier, max-over-ranks timing, the default kv-head split of one
sequence (each rank's inputs are its heads' slice, the slices tile the
sequence's heads) and the per-rank independent sequence of the replica mode;
no collective on the data path."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    import torch.distributed as dist
    from long_context_sparse_apb_b200 import inputs

    w, r, _ = bench.dist_setup(world)
    assert (w, r) == (world, rank)
    bench.barrier(w)
    mx = bench.max_over_ranks(10.0 + rank, w)
    cfg = bench.rank_config(inputs.TINY, r)
    lcfg, lx = bench.local_work(inputs.TINY, "heads", r, w)
    assert (lcfg.n_kv_heads, lcfg.n_q_heads) == (1, 2)
    out.put((rank, mx, cfg.seed, lx["q"].float().numpy(), lx["k"].float().numpy(),
             lx["w1"].numpy()))
    dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        # read before joining: a child holding unsent queue data cannot exit
        res = sorted((q.get(timeout=120) for _ in range(2)), key=lambda t: t[0])
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert [t[1] for t in res] == [11.0, 11.0]             # max over ranks
    seeds = [t[2] for t in res]
    assert seeds[0] != seeds[1]                             # independent sequences
    from long_context_sparse_apb_b200 import inputs
    full = inputs.generate(inputs.TINY)
    import numpy as np
    assert np.array_equal(np.concatenate([res[0][3], res[1][3]], axis=1), full["q"].float().numpy())
    assert np.array_equal(np.concatenate([res[0][4], res[1][4]], axis=1), full["k"].float().numpy())
    assert np.array_equal(np.concatenate([res[0][5], res[1][5]], axis=0), full["w1"].numpy())

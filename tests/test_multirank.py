"""bench.py's multi-rank plumbing on CPU ranks (gloo, world size 2): rank
setup, barrier, max-over-ranks timing and the per-rank independent sequence
(weak scaling, no collective on the data path)."""
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
    out.put((rank, mx, cfg.seed))
    dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [m for _, m, _ in res] == [11.0, 11.0]          # max over ranks
    seeds = [s for _, _, s in res]
    assert seeds[0] != seeds[1]                             # independent sequences

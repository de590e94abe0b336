"""The all-gather of the host-sharded prefill on CPU ranks (gloo, world
size 2): every rank ends with all ranks' compressed-block rows in host order,
and the host ranges partition the hosts."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from long_context_sparse_apb_b200.sharded import host_range


def test_host_ranges_partition():
    for H, W in ((8, 1), (8, 2), (8, 4), (8, 8), (16, 8)):
        got = [host_range(H, r, W) for r in range(W)]
        assert got[0][0] == 0 and got[-1][1] == H
        assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
    with pytest.raises(ValueError):
        host_range(8, 0, 3)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    from long_context_sparse_apb_b200.sharded import host_range, list_all_gather

    dist.init_process_group("gloo")
    H, keep, hkv, d = 4, 3, 2, 4
    full = torch.zeros(H * keep, hkv, d)
    hb, he = host_range(H, rank, world)
    for h in range(hb, he):                 # this rank's compressed blocks
        full[h * keep:(h + 1) * keep] = 100 * h + torch.arange(keep * hkv * d).reshape(keep, hkv, d)
    list_all_gather()(full, full[hb * keep:he * keep])
    q.put((rank, full.numpy()))
    dist.destroy_process_group()


def test_exchange_two_gloo_ranks():
    import torch
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = dict(q.get(timeout=5) for _ in range(2))
    keep, hkv, d = 3, 2, 4
    expect = torch.cat([100 * h + torch.arange(keep * hkv * d).reshape(keep, hkv, d)
                        for h in range(4)]).float()
    for r in range(2):
        assert torch.equal(torch.from_numpy(res[r]), expect)

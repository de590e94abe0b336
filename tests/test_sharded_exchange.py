"""The all-gather of the host-sharded prefill on CPU ranks (gloo, world
size 2): ShardedPrefill.exchange, with the same all_gather_into_tensor call
the GPU ranks make over NCCL, leaves every rank with all ranks'
compressed-block rows in host order, for both host assignments; the host
sets partition the hosts."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from long_context_sparse_apb_b200.sharded import exchange_chunks, host_range, host_set


def test_host_ranges_partition():
    for H, W in ((8, 1), (8, 2), (8, 4), (8, 8), (16, 8)):
        got = [host_range(H, r, W) for r in range(W)]
        assert got[0][0] == 0 and got[-1][1] == H
        assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
    with pytest.raises(ValueError):
        host_range(8, 0, 3)


@pytest.mark.parametrize("order", ["round_robin", "contiguous"])
def test_host_sets_partition_and_chunks_tile_the_buffer(order):
    for H, W, keep in ((8, 1, 3), (8, 2, 3), (8, 4, 2), (8, 8, 1), (16, 4, 5)):
        owned = []
        for r in range(W):
            first, count, stride = host_set(H, r, W, order)
            owned += [first + i * stride for i in range(count)]
            for full, chunk in exchange_chunks(H, keep, r, W, order):
                # each rank's chunk is its slot `r` of an all-gather over `full`
                assert full.stop - full.start == W * (chunk.stop - chunk.start)
                assert chunk.start - full.start == r * (chunk.stop - chunk.start)
                hosts = range(chunk.start // keep, chunk.stop // keep)
                assert all((h - first) % stride == 0 and 0 <= (h - first) // stride < count
                           for h in hosts)          # a rank sends only its own hosts' rows
        assert sorted(owned) == list(range(H))
    # round-robin balances work that grows linearly with the host index
    def spread(order, H=8, W=2):
        loads = []
        for r in range(W):
            first, count, stride = host_set(H, r, W, order)
            loads.append(sum(1 + first + i * stride for i in range(count)))
        return max(loads) - min(loads)
    assert spread("round_robin") < spread("contiguous")

def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q, order):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import datetime

    import torch
    import torch.distributed as dist
    from long_context_sparse_apb_b200 import _lib as apb
    from long_context_sparse_apb_b200.sharded import ShardedPrefill, tensor_all_gather

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    H, n, keep, hkv, d = 4, 16, 3, 2, 64
    c = apb.make_config(None, n_hosts=H, block_len=n, anchor_len=4, query_len=2, keep=keep,
                        n_q_heads=4, n_kv_heads=hkv, head_dim=d)
    # the exchange of the GPU path (all_gather_into_tensor on slices of the
    # passing buffers), run on CPU tensors between gloo ranks
    sp = ShardedPrefill(c, rank, world, device="cpu", all_gather=tensor_all_gather(), order=order)
    sp.pass_k.zero_()
    sp.pass_v.zero_()
    for h in sp.hosts:                                         # this rank's blocks
        blk = 100 * h + torch.arange(keep * hkv * d).reshape(keep, hkv, d)
        sp.pass_k[h * keep:(h + 1) * keep] = blk.to(torch.bfloat16)
        sp.pass_v[h * keep:(h + 1) * keep] = (-blk).to(torch.bfloat16)
    sp.exchange()
    q.put((rank, sp.pass_k.float().numpy(), sp.pass_v.float().numpy()))
    dist.destroy_process_group()


@pytest.mark.parametrize("order", ["round_robin", "contiguous"])
def test_exchange_two_gloo_ranks(order):
    import torch
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, order)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        # read before joining: a child holding unsent queue data cannot exit
        res = {r: (k, v) for r, k, v in (q.get(timeout=120) for _ in range(2))}
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    keep, hkv, d = 3, 2, 64
    expect = torch.cat([100 * h + torch.arange(keep * hkv * d).reshape(keep, hkv, d)
                        for h in range(4)]).to(torch.bfloat16).float()
    for r in range(2):
        assert torch.equal(torch.from_numpy(res[r][0]), expect)
        assert torch.equal(torch.from_numpy(res[r][1]), -expect)

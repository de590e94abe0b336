"""Host-sharded prefill (several GPUs in the pages' design) emulated on one
GPU: W ranks run their steps on their own rank-local buffers, the all-gather
of the compressed blocks is emulated by copying each rank's chunk into every
rank's passing buffer.  Each rank's output is checked against the fp64
oracle (selection within the tie rule, attention within the stated
tolerance on the ranks' own index set) and against the single-GPU path bit
for bit (same kernels, same arithmetic per tile).  Likewise for the
kv-head split."""
import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_apb_b200 import inputs

from _parity import check_topk, compare_attention, f32np, oracle_scores


def _oracle_check(cfg, x, idx_all, out_of_host, heads=None):
    """idx_all [H, Hkv, keep] global positions chosen by the GPU ranks;
    out_of_host(h) -> the ranks' output rows of host h [n, nh, d] (heads
    `heads`, default all)."""
    if cfg.keep > 0:
        check_topk(idx_all, oracle_scores(cfg, x), cfg)
    k, v = f32np(x["k"]), f32np(x["v"])
    pk, pv = oracle.passing_blocks(k, v, idx_all.astype(np.int64))
    n = cfg.block_len
    for h in range(cfg.n_hosts):
        o_ref, _, _ = oracle.host_attention(f32np(x["q"][h * n:(h + 1) * n]), np.arange(n), h, k,
                                            v, pk, pv, n, cfg.anchor_len, cfg.keep, heads=heads)
        compare_attention(f32np(out_of_host(h)), o_ref, f"{cfg.name} host {h}")

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("order", ["round_robin", "contiguous"])
@pytest.mark.parametrize("cfg,world", [
    (inputs.TINY, 2), (inputs.TINY, 4),
    (inputs.TINY.replace(n_hosts=6, block_len=300, anchor_len=75, keep=50, n_q_heads=8,
                         head_dim=128, seed=21), 3),
], ids=["tiny_w2", "tiny_w4", "ragged_w3"])
def test_sharded_equals_single_gpu(cfg, world, order):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_apb_b200 import _lib as apb
    from long_context_sparse_apb_b200.sharded import ShardedPrefill, exchange_chunks

    x = inputs.generate(cfg)
    c = apb.make_config(cfg)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    ref = apb.Prefill(c)(xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"], xd["b2"]).clone()

    ranks, locs = [], []
    for r in range(world):
        sp = ShardedPrefill(c, r, world, order=order)
        loc = {k: v.cuda() for k, v in inputs.generate_local(
            cfg, sp.first, sp.first + sp.count * sp.stride, sp.stride).items()}
        sp.compress(loc["q"], loc["k"], loc["v"], loc["w1"], loc["b1"], loc["w2"], loc["b2"])
        ranks.append(sp)
        locs.append(loc)
    keep = cfg.keep
    for r, src in enumerate(ranks):         # the all-gathers, emulated
        for _, rows in exchange_chunks(cfg.n_hosts, keep, r, world, order):
            for dst in ranks:
                if dst is not src:
                    dst.pass_k[rows].copy_(src.pass_k[rows])
                    dst.pass_v[rows].copy_(src.pass_v[rows])
    n = cfg.block_len
    rows_of_host = {}
    idx_all = np.zeros((cfg.n_hosts, cfg.n_kv_heads, keep), dtype=np.int64)
    for sp, loc in zip(ranks, locs):
        out = sp.attend(loc["q"], loc["k"], loc["v"])
        torch.cuda.synchronize()
        assert apb.device_status(sp.workspace) == apb.APB_OK
        for i, h in enumerate(sp.hosts):
            assert torch.equal(out[i * n:(i + 1) * n], ref[h * n:(h + 1) * n]), (order, h)
            rows_of_host[h] = out[i * n:(i + 1) * n].clone()
            idx_all[h] = sp.idx[i, 0].cpu().numpy() + h * n      # one-host calls: local rows
    _oracle_check(cfg, x, idx_all, lambda h: rows_of_host[h])


@pytest.mark.parametrize("world", [2])
def test_kv_head_sharding_equals_single_gpu(world):
    # kv-head partitioning: each rank runs the whole path on its kv heads and
    # their q heads; the outputs are the matching head slices of the full run
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_apb_b200 import _lib as apb
    from long_context_sparse_apb_b200.sharded import head_slice, kv_head_range

    cfg = inputs.TINY
    x = inputs.generate(cfg)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    full = apb.Prefill(apb.make_config(cfg))
    ref = full(xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"], xd["b2"]).clone()
    G = cfg.group
    n, H = cfg.block_len, cfg.n_hosts
    outs, idx_all = [], np.zeros((H, cfg.n_kv_heads, cfg.keep), dtype=np.int64)
    for r in range(world):
        gb, ge = kv_head_range(cfg.n_kv_heads, r, world)
        loc = head_slice(xd, cfg.n_q_heads, cfg.n_kv_heads, gb, ge)
        c = apb.make_config(cfg, n_q_heads=(ge - gb) * G, n_kv_heads=ge - gb)
        run = apb.Prefill(c)
        out = run(loc["q"], loc["k"], loc["v"], loc["w1"], loc["b1"], loc["w2"], loc["b2"])
        torch.cuda.synchronize()
        assert torch.equal(out, ref[:, gb * G:ge * G])
        assert torch.equal(run.idx, full.idx[:, gb:ge])
        outs.append(out.clone())
        # the one-call path compresses hosts 0..H-2 only (the last host's
        # block has no reader); the oracle check needs every host's indices
        idx_all[:H - 1, gb:ge] = run.idx[:H - 1].cpu().numpy()
    sh = torch.cat(outs, dim=1)               # heads back in order
    s_ref = oracle_scores(cfg, x)
    idx_all[H - 1] = oracle.compress_indices(s_ref, H, n, cfg.keep)[H - 1]
    _oracle_check(cfg, x, idx_all, lambda h: sh[h * n:(h + 1) * n])

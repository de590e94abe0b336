"""Full-size workloads (32K-512K) in the launch configuration bench.py times.

Scores, top-k and the passing block are compared on every element; attention
on seeded row samples per host (the sequence edges, the anchor's last row and
the first tile boundary are always included): all q heads on the edge rows,
and one or two q heads on the rest of the sample.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_apb_b200 import inputs

from _parity import check_topk, compare_attention, f32np, oracle_scores, SCORE_ABS

pytestmark = pytest.mark.gpu

WORKLOADS = ["llama8b_32k", "llama8b_128k", "qwen14b_128k", "llama8b_1m_512k"]


@pytest.fixture(scope="module")
def apb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_apb_b200 import _lib
    return _lib


@pytest.mark.parametrize("name", WORKLOADS)
def test_full_size_workload(apb, name):
    cfg = inputs.CONFIGS[name]
    x = inputs.generate(cfg)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    c = apb.make_config(cfg)
    run = apb.Prefill(c)
    scores = torch.empty((cfg.n_kv_heads, cfg.seq_len), dtype=torch.float32, device="cuda")
    apb.score_compress(c, xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"], xd["b2"],
                       scores=scores, idx=run.idx, workspace=run.workspace)
    out = run(xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"], xd["b2"])
    torch.cuda.synchronize()
    assert apb.device_status(run.workspace) == apb.APB_OK
    idx = run.idx.cpu().numpy()
    del xd

    s_ref = oracle_scores(cfg, x)
    assert np.abs(scores.cpu().numpy() - s_ref).max() <= SCORE_ABS
    check_topk(idx, s_ref, cfg)
    k16, v16 = x["k"].view(torch.int16).numpy(), x["v"].view(torch.int16).numpy()
    rk, rv = oracle.passing_blocks(k16, v16, idx.astype(np.int64))
    pk16 = run.pass_k.view(torch.int16).permute(1, 0, 2).cpu().numpy()
    pv16 = run.pass_v.view(torch.int16).permute(1, 0, 2).cpu().numpy()
    assert np.array_equal(pk16, rk) and np.array_equal(pv16, rv)

    k, v = f32np(x["k"]), f32np(x["v"])
    pkn = f32np(run.pass_k.permute(1, 0, 2).cpu())
    pvn = f32np(run.pass_v.permute(1, 0, 2).cpu())
    n, G = cfg.block_len, cfg.group
    nrows = cfg.sample_rows_per_host or 512
    for h in range(cfg.n_hosts):
        rows = inputs.sample_rows(cfg, h, nrows).numpy()
        edge = np.array(sorted({0, n - 1, 127, 128, cfg.anchor_len - 1} & set(range(n))))
        q_h = x["q"][h * n:(h + 1) * n]
        o_gpu_h = out[h * n:(h + 1) * n]
        # all heads on the edge rows
        o_ref, _, _ = oracle.host_attention(f32np(q_h[edge]), edge, h, k, v, pkn, pvn, n,
                                            cfg.anchor_len, cfg.keep)
        compare_attention(o_gpu_h[edge].float().cpu().numpy(), o_ref, f"{name} h{h} edge")
        heads = [(5 * h + 1) % cfg.n_q_heads]
        if cfg.sample_rows_per_host is None:
            heads.append((heads[0] + 3 * G) % cfg.n_q_heads)
        o_ref, _, _ = oracle.host_attention(f32np(q_h[rows]), rows, h, k, v, pkn, pvn, n,
                                            cfg.anchor_len, cfg.keep, heads=heads)
        got = o_gpu_h[torch.as_tensor(rows, device=out.device)][:, heads].float().cpu().numpy()
        compare_attention(got, o_ref, f"{name} h{h} sample")


@pytest.mark.parametrize("name", ["llama8b_32k", "llama8b_128k"])
def test_full_size_query_aware_selection(apb, name):
    from _parity import oracle_scores_query_aware
    cfg = inputs.CONFIGS[name]
    x = inputs.generate(cfg)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    c = apb.make_config(cfg)
    scores = torch.empty((cfg.n_kv_heads, cfg.seq_len), dtype=torch.float32, device="cuda")
    ws = apb.new_workspace(c)
    idx, _ = apb.score_compress(c, xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"],
                                xd["b2"], scores=scores, workspace=ws, query_aware=True)
    torch.cuda.synchronize()
    assert apb.device_status(ws) == apb.APB_OK
    s_ref = oracle_scores_query_aware(cfg, x)
    assert np.abs(scores.cpu().numpy() - s_ref).max() <= SCORE_ABS
    check_topk(idx.cpu().numpy(), s_ref, cfg)

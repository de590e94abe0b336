"""CUDA path (through the C ABI) against the fp64 CPU oracle.

* scores: fp32 GPU vs fp64 oracle within SCORE_ABS;
* top-k: identical sets except swaps within a 1e-5 relative score gap of the
  keep-th largest oracle score; ascending, in range, deterministic;
* passing block: bit-exact against the oracle's gather of the GPU's indices;
* attention: max-abs <= 2e-2 and mean-abs <= 2e-3 against the oracle run on
  the GPU's own index set (so a legal tie swap is not penalised).

Small shapes are compared element by element on every row; the full-size
workloads run in the launch configuration of bench.py and are compared on
seeded row samples (edge rows always included).
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_apb_b200 import inputs

from _parity import (check_topk, compare_attention, f32np, oracle_scores, SCORE_ABS)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def apb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_apb_b200 import _lib
    return _lib


def _to_dev(x):
    return {k: (v.cuda() if k != "needles" else v) for k, v in x.items()}


def _run_gpu(apb, cfg, xd):
    c = apb.make_config(cfg)
    N = cfg.seq_len
    scores = torch.empty((cfg.n_kv_heads, N), dtype=torch.float32, device="cuda")
    ws = apb.new_workspace(c)
    idx, _ = apb.score_compress(c, xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"],
                                xd["b2"], scores=scores, workspace=ws)
    pk, pv = apb.build_passing(c, xd["k"], xd["v"], idx)
    out, lse = apb.block_attention(c, xd["q"], xd["k"], xd["v"], pk, pv, want_lse=True,
                                   workspace=ws)
    torch.cuda.synchronize()
    assert apb.device_status(ws) == apb.APB_OK
    return scores, idx, pk, pv, out, lse


def _check_passing_exact(x, idx_np, pk, pv):
    k16 = x["k"].view(torch.int16).numpy()
    v16 = x["v"].view(torch.int16).numpy()
    rk, rv = oracle.passing_blocks(k16, v16, idx_np.astype(np.int64))
    # device layout [H*keep, Hkv, d]; the oracle's [Hkv, H*keep, d]
    assert np.array_equal(pk.view(torch.int16).permute(1, 0, 2).cpu().numpy(), rk)
    assert np.array_equal(pv.view(torch.int16).permute(1, 0, 2).cpu().numpy(), rv)


def _full_parity(apb, cfg, x=None):
    x = inputs.generate(cfg) if x is None else x
    xd = _to_dev(x)
    scores, idx, pk, pv, out, lse = _run_gpu(apb, cfg, xd)
    s_ref = oracle_scores(cfg, x)
    assert np.abs(scores.cpu().numpy() - s_ref).max() <= SCORE_ABS
    idx_np = idx.cpu().numpy()
    if cfg.keep > 0:
        check_topk(idx_np, s_ref, cfg)
    _check_passing_exact(x, idx_np, pk, pv)
    k, v = f32np(x["k"]), f32np(x["v"])
    pkn, pvn = f32np(pk.permute(1, 0, 2).cpu()), f32np(pv.permute(1, 0, 2).cpu())
    n = cfg.block_len
    o_all = out.float().cpu().numpy()
    lse_all = lse.cpu().numpy()
    for h in range(cfg.n_hosts):
        rows = np.arange(n)
        o_ref, lse_ref, _ = oracle.host_attention(f32np(x["q"][h * n:(h + 1) * n]), rows, h, k, v,
                                                  pkn, pvn, n, cfg.anchor_len, cfg.keep)
        compare_attention(o_all[h * n:(h + 1) * n], o_ref, f"{cfg.name} host {h}")
        assert np.abs(lse_all[:, h * n:(h + 1) * n].T - lse_ref).max() < 1e-3
    return out


def test_tiny_workload_every_row(apb):
    _full_parity(apb, inputs.TINY)


SMALL = [
    # H, n, A, q_len, keep, Hq, Hkv, d
    (1, 300, 64, 16, 32, 4, 2, 128),     # single host: dense causal
    (2, 128, 128, 8, 128, 2, 1, 64),     # full anchor, keep all
    (3, 100, 0, 0, 1, 4, 4, 128),        # no anchor, keep 1, n < one tile
    (5, 513, 200, 32, 0, 8, 2, 128),     # keep 0, ragged n and anchor
    (3, 257, 33, 33, 257, 10, 2, 64),    # keep = n, G = 5
    (4, 384, 96, 16, 130, 4, 1, 128),    # passing tail of 2 rows per 128-tile
    (2, 200, 50, 10, 40, 6, 2, 128),     # G = 3 (one partial head group)
    (3, 150, 40, 8, 20, 7, 1, 64),       # G = 7 (a full and a partial head group)
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
def test_small_shapes_every_row(apb, shape):
    H, n, A, ql, keep, hq, hkv, d = shape
    cfg = inputs.APBConfig("small", n_hosts=H, block_len=n, anchor_len=A, query_len=ql, keep=keep,
                           n_q_heads=hq, n_kv_heads=hkv, head_dim=d, seed=7 + H * n,
                           rope_theta=1e4, needles_per_host=2)
    _full_parity(apb, cfg)


@pytest.mark.parametrize("d,G", [(128, 4), (64, 2)])
def test_star_configuration_long_anchor(apb, d, G):
    # The Star-style mask the bench times next to APB (anchor = the whole
    # first block, no passing block), with H >= 3 and an anchor of 18 KV tiles
    # ending in a ragged one (2300 = 17 * 128 + 124): every row of every host
    cfg = inputs.APBConfig("star", n_hosts=3, block_len=2300, anchor_len=2300, query_len=64,
                           keep=0, n_q_heads=2 * G, n_kv_heads=2, head_dim=d, seed=41 + d,
                           rope_theta=5e5, needles_per_host=4)
    _full_parity(apb, cfg)


def test_deterministic_repeat(apb):
    cfg = inputs.TINY.replace(n_hosts=3, block_len=640, anchor_len=160, keep=100)
    xd = _to_dev(inputs.generate(cfg))
    a = _run_gpu(apb, cfg, xd)
    b = _run_gpu(apb, cfg, xd)
    for ta, tb in zip(a, b):
        assert torch.equal(ta, tb)


def test_dense_causal_reduction_on_gpu(apb):
    # H = 1: the kernel must equal dense causal attention (library, fp32)
    cfg = inputs.APBConfig("dense", n_hosts=1, block_len=1000, anchor_len=0, query_len=0, keep=0,
                           n_q_heads=8, n_kv_heads=2, head_dim=128, seed=3)
    x = inputs.generate(cfg)
    xd = _to_dev(x)
    c = apb.make_config(cfg)
    out, _ = apb.block_attention(c, xd["q"], xd["k"], xd["v"], None, None)
    q = xd["q"].float().permute(1, 0, 2)[None]
    k = xd["k"].float().repeat_interleave(4, dim=1).permute(1, 0, 2)[None]
    v = xd["v"].float().repeat_interleave(4, dim=1).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)[0]
    err = (out.float().permute(1, 0, 2) - ref).abs()
    assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3


def test_pipeline_matches_direct_calls(apb):
    # PrefillPipeline (pinned host buffers, overlapped copies) returns, for
    # each submitted step, exactly what the direct calls return
    cfgs = [inputs.TINY, inputs.TINY.replace(seed=5)]
    xs = [inputs.generate(c) for c in cfgs]
    c = apb.make_config(inputs.TINY)
    direct = []
    for x in xs:
        xd = _to_dev(x)
        run = apb.Prefill(c)
        direct.append(run(xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"], xd["b2"]).cpu())
    pipe = apb.PrefillPipeline(c, depth=2)
    outs = []
    for step in range(5):
        x = xs[step % 2]
        hx = {k: v.pin_memory() for k, v in x.items() if k != "needles"}
        ho = torch.empty_like(direct[0]).pin_memory()
        pipe.submit(hx, ho)
        outs.append((step % 2, ho, hx))
    pipe.synchronize()
    for which, ho, _ in outs:
        assert torch.equal(ho, direct[which])


@pytest.mark.parametrize("cfg", [inputs.TINY,
                                 inputs.TINY.replace(n_hosts=5, block_len=300, anchor_len=75,
                                                     keep=40, n_q_heads=8, head_dim=128, seed=14),
                                 inputs.TINY.replace(n_hosts=1, seed=15)],
                         ids=["tiny", "ragged_5_hosts", "one_host"])
def test_streamed_prefill_matches_direct_calls(apb, cfg):
    # StreamedPrefill (host-by-host copies, compression and attention on
    # several streams) returns, for each submitted step, exactly what the
    # three direct calls return
    cfgs = [cfg, cfg.replace(seed=cfg.seed + 100)]
    xs = [inputs.generate(k) for k in cfgs]
    c = apb.make_config(cfg)
    direct = []
    for x in xs:
        xd = _to_dev(x)
        run = apb.Prefill(c)
        direct.append(run(xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"], xd["b2"]).cpu())
    pipe = apb.StreamedPrefill(c, depth=2)
    outs = []
    for step in range(5):
        x = xs[step % 2]
        hx = {k: v.pin_memory() for k, v in x.items() if k != "needles"}
        ho = torch.empty_like(direct[0]).pin_memory()
        pipe.submit(hx, ho)
        outs.append((step % 2, ho, hx))
    pipe.synchronize()
    for ws in pipe.workspaces():
        assert apb.device_status(ws) == apb.APB_OK
    for which, ho, _ in outs:
        assert torch.equal(ho, direct[which])


@pytest.mark.parametrize("cfg", [inputs.TINY,
                                 inputs.TINY.replace(n_hosts=3, block_len=300, anchor_len=75,
                                                     query_len=0, keep=40, seed=9),
                                 inputs.TINY.replace(n_q_heads=10, n_kv_heads=2, head_dim=128,
                                                     seed=12)],
                         ids=["tiny", "no_query_segment", "g5_d128"])
def test_query_aware_scores_and_selection(apb, cfg):
    from _parity import oracle_scores_query_aware
    x = inputs.generate(cfg)
    xd = _to_dev(x)
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
    # the two variants differ (own-token q vs query-segment q) unless q_len covers nothing
    idx2, _ = apb.score_compress(c, xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"],
                                 xd["b2"], workspace=ws)
    assert idx2.shape == idx.shape


def _random_shapes(count, seed=2026):
    rng = np.random.default_rng(seed)
    shapes = [
        # degenerate cases first: one-token blocks, anchor = whole block, keep = n = 1
        (3, 1, 1, 1, 1, 2, 1, 64),
        (2, 1, 0, 0, 0, 4, 4, 128),
        (1, 5, 5, 2, 5, 8, 1, 128),          # one host, G = 8
    ]
    while len(shapes) < count:
        H = int(rng.integers(1, 6))
        n = int(rng.integers(2, 700))
        A = int(rng.integers(0, n + 1))
        ql = int(rng.integers(0, A + 1))
        keep = int(rng.choice([0, 1, int(rng.integers(1, n + 1)), n]))
        hkv = int(rng.choice([1, 2, 4]))
        G = int(rng.choice([1, 2, 4, 5, 8]))
        d = int(rng.choice([64, 128]))
        shapes.append((H, n, A, ql, keep, hkv * G, hkv, d))
    return shapes


@pytest.mark.parametrize("shape", _random_shapes(14), ids=lambda s: "x".join(map(str, s)))
def test_random_shapes_every_row(apb, shape):
    H, n, A, ql, keep, hq, hkv, d = shape
    cfg = inputs.APBConfig("rand", n_hosts=H, block_len=n, anchor_len=A, query_len=ql, keep=keep,
                           n_q_heads=hq, n_kv_heads=hkv, head_dim=d, seed=31 + H + n + keep,
                           rope_theta=1e4 if d == 128 else None, needles_per_host=1)
    _full_parity(apb, cfg)


@pytest.mark.parametrize("cfg", [inputs.TINY,
                                 inputs.TINY.replace(n_hosts=5, block_len=300, anchor_len=75,
                                                     keep=33, n_q_heads=10, head_dim=128, seed=4),
                                 inputs.TINY.replace(n_hosts=1, seed=6),
                                 inputs.TINY.replace(keep=0, seed=7)],
                         ids=["tiny", "ragged_g5", "one_host", "keep0"])
def test_single_call_prefill_equals_three_calls(apb, cfg):
    # apb_prefill skips the last host's compressed block; its output and LSE
    # must equal the three-call path's bit for bit
    x = inputs.generate(cfg)
    xd = _to_dev(x)
    c = apb.make_config(cfg)
    w = (xd["w1"], xd["b1"], xd["w2"], xd["b2"])
    run = apb.Prefill(c)
    apb.score_compress(c, xd["q"], xd["k"], xd["v"], *w, idx=run.idx, workspace=run.workspace)
    apb.build_passing(c, xd["k"], xd["v"], run.idx, run.pass_k, run.pass_v)
    ref, ref_lse = apb.block_attention(c, xd["q"], xd["k"], xd["v"], run.pass_k, run.pass_v,
                                       want_lse=True, workspace=run.workspace)
    ws = torch.zeros(apb.prefill_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    out, lse = apb.prefill(c, xd["q"], xd["k"], xd["v"], *w, want_lse=True, workspace=ws)
    torch.cuda.synchronize()
    assert apb.device_status(ws) == apb.APB_OK
    assert torch.equal(out, ref) and torch.equal(lse, ref_lse)


@pytest.mark.parametrize("cfg", [inputs.TINY,
                                 inputs.TINY.replace(n_hosts=5, block_len=300, anchor_len=75,
                                                     keep=130, n_q_heads=10, n_kv_heads=2,
                                                     head_dim=128, seed=13),
                                 inputs.TINY.replace(keep=512, seed=14),
                                 inputs.TINY.replace(n_hosts=3, block_len=1000, anchor_len=100,
                                                     keep=777, seed=15)],
                         ids=["tiny", "ragged_g5", "keep_n", "ragged_parts"])
def test_score_compress_pass_equals_separate_calls(apb, cfg):
    # selection and gather in one launch: idx, scores and both passing
    # buffers equal the two-call path bit for bit (ragged_parts: the gather
    # of each (host, kv head) split over 6 CTAs, the last with fewer rows)
    x = inputs.generate(cfg)
    xd = _to_dev(x)
    c = apb.make_config(cfg)
    N, hq, hkv, d = c.n_hosts * c.block_len, c.n_q_heads, c.n_kv_heads, c.head_dim
    w = (xd["w1"], xd["b1"], xd["w2"], xd["b2"])
    ref_scores = torch.empty((hkv, N), dtype=torch.float32, device="cuda")
    ref_idx, _ = apb.score_compress(c, xd["q"], xd["k"], xd["v"], *w, scores=ref_scores)
    ref_pk, ref_pv = apb.build_passing(c, xd["k"], xd["v"], ref_idx)
    scores = torch.empty_like(ref_scores)
    pk = torch.full_like(ref_pk, float("nan"))
    pv = torch.full_like(ref_pv, float("nan"))
    idx = apb.score_compress_pass(c, xd["q"], xd["k"], xd["v"], *w, pk, pv, scores=scores)
    torch.cuda.synchronize()
    assert torch.equal(idx, ref_idx)
    assert torch.equal(scores.view(torch.int32), ref_scores.view(torch.int32))
    assert torch.equal(pk.view(torch.int16), ref_pk.view(torch.int16))
    assert torch.equal(pv.view(torch.int16), ref_pv.view(torch.int16))


@pytest.mark.parametrize("mult", [14.0, 60.0], ids=["x_about_80", "x_about_345"])
def test_scores_far_above_the_first_tiles(apb, mult):
    # the softmax keeps the first tile's row maximum as its base and moves it
    # only when a 64-column half's probabilities would pass 2^64: plant one
    # key whose logits lie ~80 or ~345 (log2 units) above everything the rows
    # saw before, for kv head 0 in the first half of host 1's first local
    # tile and for kv head 1 in its second half, so both of those paths run
    # (the second after the first half's probabilities have gone to the
    # tensor core); at ~345 the probabilities would overflow without them
    cfg = inputs.TINY.replace(seed=41)
    x = inputs.generate(cfg)
    n, G, d = cfg.block_len, cfg.group, cfg.head_dim
    h = 1
    gen = torch.Generator().manual_seed(41)
    q = x["q"].float()
    k = x["k"].float()
    # host h's queries: one direction per q head (|u|^2 ~ d) plus a little noise
    u = torch.randn(cfg.n_q_heads, d, generator=gen)
    q[h * n:(h + 1) * n] = u[None] + 0.1 * torch.randn(n, cfg.n_q_heads, d, generator=gen)
    for g, local in ((0, 10), (1, 72)):          # local tile 0, column 10 / column 72
        ug = u[g * G:(g + 1) * G].mean(0)
        k[h * n + local, g] = mult * ug          # logit ~ mult * (d / 2) / sqrt(d) * log2(e)
    x["q"] = q.to(torch.bfloat16)
    x["k"] = k.to(torch.bfloat16)
    _full_parity(apb, cfg, x)


def test_topk_unstaged_path_large_block(apb):
    # blocks above 48K tokens re-read their scores from global memory in every
    # radix pass instead of staging them in shared memory
    cfg = inputs.APBConfig("bigblock", n_hosts=2, block_len=50_000, anchor_len=0, query_len=0,
                           keep=3000, n_q_heads=2, n_kv_heads=1, head_dim=64, seed=17)
    x = inputs.generate(cfg)
    xd = _to_dev(x)
    c = apb.make_config(cfg)
    scores = torch.empty((1, cfg.seq_len), dtype=torch.float32, device="cuda")
    idx, _ = apb.score_compress(c, xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"],
                                xd["b2"], scores=scores)
    pk, pv = apb.build_passing(c, xd["k"], xd["v"], idx)
    torch.cuda.synchronize()
    s_ref = oracle_scores(cfg, x)
    assert np.abs(scores.cpu().numpy() - s_ref).max() <= SCORE_ABS
    check_topk(idx.cpu().numpy(), s_ref, cfg)
    _check_passing_exact(x, idx.cpu().numpy(), pk, pv)
    # the fused form on the same path: each (host, kv head) split over many
    # CTAs (2 units, 3000 rows), every one re-reading the scores from global
    # memory; bit-equal to the two calls
    pk2 = torch.full_like(pk, float("nan"))
    pv2 = torch.full_like(pv, float("nan"))
    idx2 = apb.score_compress_pass(c, xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"],
                                   xd["b2"], pk2, pv2)
    torch.cuda.synchronize()
    assert torch.equal(idx2, idx)
    assert torch.equal(pk2.view(torch.int16), pk.view(torch.int16))
    assert torch.equal(pv2.view(torch.int16), pv.view(torch.int16))

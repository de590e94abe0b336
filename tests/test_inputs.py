"""Seeded synthetic inputs: shapes, determinism and the planted needles."""
import math

import torch

from long_context_sparse_apb_b200 import inputs


def test_tiny_shapes_and_determinism():
    cfg = inputs.TINY
    a = inputs.generate(cfg)
    b = inputs.generate(cfg)
    N = cfg.seq_len
    assert a["q"].shape == (N, cfg.n_q_heads, cfg.head_dim) and a["q"].dtype == torch.bfloat16
    assert a["k"].shape == (N, cfg.n_kv_heads, cfg.head_dim)
    assert a["w1"].shape == (cfg.n_kv_heads, cfg.mlp_hidden, 3 * cfg.head_dim)
    assert a["w1"].dtype == torch.float32
    for key in ("q", "k", "v", "w1", "b1", "w2", "b2", "needles"):
        assert torch.equal(a[key], b[key]), key
    assert abs(a["w1"].std().item() - 0.02) < 2e-3


def test_needles_planted_outside_anchor():
    cfg = inputs.TINY
    x = inputs.generate(cfg)
    pos = x["needles"]
    assert pos.numel() == cfg.n_hosts * cfg.needles_per_host
    assert torch.all(pos >= cfg.anchor_len)
    for h in range(cfg.n_hosts):
        ph = pos[(pos >= h * cfg.block_len) & (pos < (h + 1) * cfg.block_len)]
        assert ph.numel() == cfg.needles_per_host
    norms = x["k"][pos].float().norm(dim=-1)
    assert torch.allclose(norms, torch.full_like(norms, 3 * math.sqrt(cfg.head_dim)), rtol=1e-2)


def test_sample_rows_hold_edges():
    cfg = inputs.LLAMA8B_1M_512K
    r = inputs.sample_rows(cfg, 3, 4096)
    assert r.numel() == 4096
    assert torch.all(r[1:] > r[:-1])
    for must in (0, cfg.block_len - 1, cfg.anchor_len - 1, 127, 128):
        assert must in r.tolist()


def test_generate_local_matches_full_sequence():
    cfg = inputs.TINY
    x = inputs.generate(cfg)
    n, A = cfg.block_len, cfg.anchor_len
    for hb, he in ((0, 2), (2, 4), (1, 4), (3, 4)):
        loc = inputs.generate_local(cfg, hb, he)
        assert torch.equal(loc["q"], x["q"][hb * n:he * n])
        for t in ("k", "v"):
            assert torch.equal(loc[t][:A], x[t][:A])
            assert torch.equal(loc[t][A:], x[t][hb * n:he * n])
        assert torch.equal(loc["w1"], x["w1"])

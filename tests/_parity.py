"""Helpers of the GPU-vs-oracle parity tests (test infrastructure)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from long_context_sparse_apb_b200 import inputs

ATTN_MAX_ABS = 2e-2       # bf16 output vs the fp64 oracle
ATTN_MEAN_ABS = 2e-3
TIE_REL = 1e-5            # top-k swaps allowed only within this relative score gap
SCORE_ABS = 2e-5          # fp32 GPU scores vs fp64 oracle (scores are O(0.1-1))


def f32np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def oracle_scores(cfg: inputs.APBConfig, x) -> np.ndarray:
    """fp64 oracle scores [Hkv, N], computed host block by host block."""
    n = cfg.block_len
    out = np.empty((cfg.n_kv_heads, cfg.seq_len), dtype=np.float64)
    w = [x[k].numpy() for k in ("w1", "b1", "w2", "b2")]
    for h in range(cfg.n_hosts):
        sl = slice(h * n, (h + 1) * n)
        out[:, sl] = oracle.retaining_scores(f32np(x["q"][sl]), f32np(x["k"][sl]),
                                             f32np(x["v"][sl]), *w)
    return out


def check_topk(idx_gpu: np.ndarray, s_ref: np.ndarray, cfg, tie_rel=TIE_REL) -> int:
    """Selected sets must equal the oracle's except for swaps whose scores are
    within tie_rel of the keep-th largest oracle score.  Returns the number of
    (host, kv head) units whose sets differ (legally)."""
    H, hkv, keep = idx_gpu.shape
    n = cfg.block_len
    idx_ref = oracle.compress_indices(s_ref, H, n, keep)
    differing = 0
    for h in range(H):
        for g in range(hkv):
            got = idx_gpu[h, g].astype(np.int64)
            assert np.all(np.diff(got) > 0), f"idx not strictly ascending at h={h} g={g}"
            assert got.min(initial=h * n) >= h * n and got.max(initial=h * n) < (h + 1) * n
            ref = idx_ref[h, g]
            if np.array_equal(got, ref):
                continue
            differing += 1
            seg = s_ref[g, h * n:(h + 1) * n]
            kth = np.sort(seg)[::-1][keep - 1]
            swapped = np.setxor1d(got, ref)
            gap = np.abs(s_ref[g, swapped] - kth)
            assert np.all(gap <= tie_rel * abs(kth)), (
                f"top-k differs beyond ties at h={h} g={g}: gaps {gap.max():.3e} vs "
                f"{tie_rel * abs(kth):.3e}")
    return differing


def oracle_rows(cfg, x, pass_k, pass_v, host, rows, heads=None):
    """fp64 oracle attention for some rows of one host (oracle passing block
    given as numpy, built from the GPU's own index set)."""
    n = cfg.block_len
    q = x["q"]
    qr = f32np(q[host * n + torch.as_tensor(rows)])
    return oracle.host_attention(qr, rows, host, x["k_np"], x["v_np"], pass_k, pass_v, n,
                                 cfg.anchor_len, cfg.keep, heads=heads)


def compare_attention(o_gpu: np.ndarray, o_ref: np.ndarray, what: str):
    err = np.abs(o_gpu.astype(np.float64) - o_ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def oracle_scores_query_aware(cfg: inputs.APBConfig, x) -> np.ndarray:
    """fp64 oracle of the query-aware score variant [Hkv, N]."""
    n = cfg.block_len
    out = np.empty((cfg.n_kv_heads, cfg.seq_len), dtype=np.float64)
    w = [x[k].numpy() for k in ("w1", "b1", "w2", "b2")]
    q_seg = f32np(x["q"][:cfg.query_len])
    for h in range(cfg.n_hosts):
        sl = slice(h * n, (h + 1) * n)
        out[:, sl] = oracle.retaining_scores_query_aware(q_seg, f32np(x["k"][sl]),
                                                         f32np(x["v"][sl]), *w)
    return out

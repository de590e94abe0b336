"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each check is chosen so that a plausible slip in the oracle (a dropped bias, a
wrong group mapping, an off-by-one in the anchor or causal range, the wrong
host prefix for the passing block, a wrong tie rule) fails at least one:

* score: closed-form SiLU values on a hand-built case (feature order k, v,
  mean_group(q); both biases; the group mean);
* top-k: brute-force rank counting on small inputs; constructed ties;
* passing block: its definition row by row, and the all-kept reduction;
* attention: reductions to dense causal attention computed by
  ``torch.nn.functional.scaled_dot_product_attention`` in float64
  (H = 1; keep = n with no anchor; a full-block anchor with keep = 0; host 0
  of any configuration), an additive-bias identity for duplicated keys,
  softmax normalisation and invariance to the passing block's row order;
* visible-pair count: an explicit per-slot visibility mask on tiny cases, and
  the number of keys the oracle's attention spreads its weight over.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import (compress_indices, host_attention, passing_blocks, retaining_scores_query_aware,
                    retaining_scores, visible_pairs)
from long_context_sparse_apb_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _dense_causal(q, k, v):
    """Library dense causal attention, float64. q [N,Hq,d], k/v [N,Hkv,d]."""
    hq, hkv = q.shape[1], k.shape[1]
    G = hq // hkv
    qt = torch.as_tensor(np.asarray(q, np.float64)).permute(1, 0, 2)[None]
    kt = torch.as_tensor(np.asarray(k, np.float64)).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    vt = torch.as_tensor(np.asarray(v, np.float64)).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    return o[0].permute(1, 0, 2).numpy()


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _full_host_rows(q, host, n):
    return q[host * n:(host + 1) * n], np.arange(n)


# ----------------------------------------------------------------- score

def test_score_closed_form_golden():
    g = json.load(open(os.path.join(GOLDEN, "score_closed_form.json")))
    ln3, s3, e = math.log(3.0), math.sqrt(3.0), math.e
    q = np.array(g["q"])
    k = np.array(g["k"])
    v = np.array(g["v"])
    w1 = np.zeros((1, 3, 6))
    w1[0, 0, 0] = ln3            # k[0]
    w1[0, 1, 3] = -ln3 / 2       # v[1]
    w1[0, 2, 5] = 1.0            # qbar[1]
    b1 = np.array([[0.0, 0.0, -2.0]])
    w2 = np.array(g["w2"])
    b2 = np.array(g["b2"])
    s = retaining_scores(q, k, v, w1, b1, w2, b2)
    expect = [ln3 / 4 + 0.25, 1.8 * ln3 + ln3 * s3 / (s3 + 1) + 5 * e / (e + 1) + 0.25]
    assert s.shape == (1, 2)
    np.testing.assert_allclose(s[0], expect, rtol=0, atol=1e-14)


def test_score_group_mapping_consecutive():
    # 4 q heads, 2 kv heads: kv head 0 must average q heads {0,1}, kv head 1 {2,3}
    d, T = 3, 2
    q = np.zeros((T, 4, d))
    q[:, 0, 0], q[:, 1, 0], q[:, 2, 0], q[:, 3, 0] = 1.0, 3.0, 10.0, 30.0
    k = np.zeros((T, 2, d))
    v = np.zeros((T, 2, d))
    w1 = np.zeros((2, 1, 3 * d))
    w1[:, 0, 2 * d] = 1.0        # hidden unit = qbar[0]
    b1 = np.zeros((2, 1))
    w2 = np.ones((2, 1))
    b2 = np.zeros(2)
    s = retaining_scores(q, k, v, w1, b1, w2, b2)
    silu = lambda z: z / (1 + math.exp(-z))
    np.testing.assert_allclose(s[0], silu(2.0), atol=1e-14)
    np.testing.assert_allclose(s[1], silu(20.0), atol=1e-12)


def test_score_linearity_in_w2_b2():
    # s is affine in (w2, b2): doubling w2 and b2 doubles s
    rng_q = _rand((5, 4, 8), 1)
    k, v = _rand((5, 2, 8), 2), _rand((5, 2, 8), 3)
    w1, b1 = _rand((2, 16, 24), 4, 0.1), _rand((2, 16), 5, 0.1)
    w2, b2 = _rand((2, 16), 6, 0.1), _rand((2,), 7, 0.1)
    s1 = retaining_scores(rng_q, k, v, w1, b1, w2, b2)
    s2 = retaining_scores(rng_q, k, v, w1, b1, 2 * w2, 2 * b2)
    np.testing.assert_allclose(s2, 2 * s1, rtol=1e-13, atol=1e-15)


# ----------------------------------------------------------------- top-k

def _brute_topk(seg, keep):
    """Token t is kept iff fewer than `keep` tokens beat it (higher score, or
    equal score at a lower position)."""
    n = len(seg)
    out = []
    for t in range(n):
        beaten_by = sum(1 for u in range(n)
                        if seg[u] > seg[t] or (seg[u] == seg[t] and u < t))
        if beaten_by < keep:
            out.append(t)
    return np.array(out, dtype=np.int64)


@pytest.mark.parametrize("H,n,keep,seed", [(1, 7, 3, 0), (3, 9, 4, 1), (2, 12, 0, 2),
                                            (2, 12, 12, 3), (4, 5, 1, 4)])
def test_topk_brute_force(H, n, keep, seed):
    s = _rand((2, H * n), seed)
    idx = compress_indices(s, H, n, keep)
    assert idx.shape == (H, 2, keep)
    for h in range(H):
        for g in range(2):
            ref = _brute_topk(s[g, h * n:(h + 1) * n], keep) + h * n
            np.testing.assert_array_equal(idx[h, g], ref)


def test_topk_ties_lower_position_wins():
    s = np.array([[0.5, 1.0, 1.0, 0.2, 1.0, 1.0]])
    idx = compress_indices(s, 1, 6, 3)
    np.testing.assert_array_equal(idx[0, 0], [1, 2, 4])
    # quantised scores: many ties, compared with the brute force rule
    q = np.round(_rand((1, 40), 9) * 2) / 2
    idx = compress_indices(q, 2, 20, 7)
    for h in range(2):
        np.testing.assert_array_equal(idx[h, 0], _brute_topk(q[0, h * 20:(h + 1) * 20], 7) + h * 20)


def test_topk_in_range_ascending_exact_count():
    s = _rand((3, 8 * 33), 11)
    idx = compress_indices(s, 8, 33, 10)
    for h in range(8):
        assert np.all(idx[h] >= h * 33) and np.all(idx[h] < (h + 1) * 33)
        assert np.all(np.diff(idx[h], axis=1) > 0)


# ----------------------------------------------------------------- passing

def test_passing_rows_follow_definition():
    H, n, keep, hkv, d = 4, 10, 3, 2, 5
    k, v = _rand((H * n, hkv, d), 1), _rand((H * n, hkv, d), 2)
    idx = compress_indices(_rand((hkv, H * n), 3), H, n, keep)
    pk, pv = passing_blocks(k, v, idx)
    assert pk.shape == (hkv, H * keep, d)
    for g in range(hkv):
        for r in range(H * keep):
            t = idx[r // keep, g, r % keep]
            assert (t // n) == r // keep                     # host order
            np.testing.assert_array_equal(pk[g, r], k[t, g])
            np.testing.assert_array_equal(pv[g, r], v[t, g])
    # host h's passing block = rows [0, h*keep): exactly the preceding hosts
    for h in range(H):
        rows = idx[:h, 0, :].reshape(-1)
        assert sorted(set(rows // n)) == list(range(h))


def test_passing_keep_all_is_whole_prefix():
    H, n, hkv, d = 3, 6, 1, 4
    k, v = _rand((H * n, hkv, d), 5), _rand((H * n, hkv, d), 6)
    idx = compress_indices(_rand((hkv, H * n), 7), H, n, n)
    pk, _ = passing_blocks(k, v, idx)
    np.testing.assert_array_equal(pk[0], k[:, 0])


# ----------------------------------------------------------------- attention

def _all_hosts(q, k, v, pk, pv, H, n, A, keep, heads=None):
    outs = []
    for h in range(H):
        qr, rows = _full_host_rows(q, h, n)
        o, _, rs = host_attention(qr, rows, h, k, v, pk, pv, n, A, keep, heads=heads)
        outs.append(o)
        np.testing.assert_allclose(rs, 1.0, atol=1e-12)
    return np.concatenate(outs, axis=0)


def test_single_host_is_dense_causal():
    n, hq, hkv, d = 200, 4, 2, 16
    q, k, v = _rand((n, hq, d), 1), _rand((n, hkv, d), 2), _rand((n, hkv, d), 3)
    pk = np.zeros((hkv, 17, d))
    o = _all_hosts(q, k, v, pk, pk, 1, n, 50, 17)
    np.testing.assert_allclose(o, _dense_causal(q, k, v), atol=1e-12)


def test_keep_all_no_anchor_is_dense_causal():
    H, n, hq, hkv, d = 3, 40, 4, 2, 8
    N = H * n
    q, k, v = _rand((N, hq, d), 4), _rand((N, hkv, d), 5), _rand((N, hkv, d), 6)
    idx = compress_indices(_rand((hkv, N), 7), H, n, n)
    pk, pv = passing_blocks(k, v, idx)
    o = _all_hosts(q, k, v, pk, pv, H, n, 0, n)
    np.testing.assert_allclose(o, _dense_causal(q, k, v), atol=1e-12)


def test_full_anchor_two_hosts_is_dense_causal():
    # H = 2, A = n, keep = 0: host 1 sees all of host 0 through the anchor
    H, n, hq, hkv, d = 2, 48, 2, 1, 8
    N = H * n
    q, k, v = _rand((N, hq, d), 8), _rand((N, hkv, d), 9), _rand((N, hkv, d), 10)
    idx = compress_indices(_rand((hkv, N), 11), H, n, 0)
    pk, pv = passing_blocks(k, v, idx)
    o = _all_hosts(q, k, v, pk, pv, H, n, n, 0)
    np.testing.assert_allclose(o, _dense_causal(q, k, v), atol=1e-12)


def test_host0_is_dense_causal_on_tiny_workload():
    cfg = inputs.TINY
    x = inputs.generate(cfg)
    q, k, v = (x[t].float().numpy() for t in ("q", "k", "v"))
    n = cfg.block_len
    s = retaining_scores(q, k, v, *(x[w].numpy() for w in ("w1", "b1", "w2", "b2")))
    idx = compress_indices(s, cfg.n_hosts, n, cfg.keep)
    pk, pv = passing_blocks(k, v, idx)
    o, _, _ = host_attention(q[:n], np.arange(n), 0, k, v, pk, pv, n, cfg.anchor_len, cfg.keep)
    np.testing.assert_allclose(o, _dense_causal(q[:n], k[:n], v[:n]), atol=1e-12)


def test_duplicated_anchor_keys_equal_log2_bias():
    # H = 2, A = n/2, keep = n: host 1 sees rows [0, n/2) twice (anchor and
    # passing).  A key present twice equals that key once with +ln 2 added to
    # its logit; check against the library routine with an additive mask.
    H, n, hq, hkv, d = 2, 32, 2, 1, 8
    N, A = H * n, 16
    q, k, v = _rand((N, hq, d), 12), _rand((N, hkv, d), 13), _rand((N, hkv, d), 14)
    idx = compress_indices(_rand((hkv, N), 15), H, n, n)
    pk, pv = passing_blocks(k, v, idx)
    o, _, _ = host_attention(q[n:], np.arange(n), 1, k, v, pk, pv, n, A, n)
    bias = np.full((N, N), -np.inf)
    for i in range(N):
        bias[i, :i + 1] = 0.0
    bias[:, :A] += math.log(2.0)
    qt = torch.as_tensor(q).permute(1, 0, 2)[None]
    kt = torch.as_tensor(k).repeat_interleave(hq // hkv, dim=1).permute(1, 0, 2)[None]
    vt = torch.as_tensor(v).repeat_interleave(hq // hkv, dim=1).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.as_tensor(bias)[None, None])[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(o, ref[n:], atol=1e-12)


def test_anchor_rows_do_not_reach_host0():
    # changing the anchor length must not change host 0 (reading R1)
    H, n, hq, hkv, d = 2, 24, 2, 2, 4
    N = H * n
    q, k, v = _rand((N, hq, d), 16), _rand((N, hkv, d), 17), _rand((N, hkv, d), 18)
    idx = compress_indices(_rand((hkv, N), 19), H, n, 5)
    pk, pv = passing_blocks(k, v, idx)
    o1, _, _ = host_attention(q[:n], np.arange(n), 0, k, v, pk, pv, n, 0, 5)
    o2, _, _ = host_attention(q[:n], np.arange(n), 0, k, v, pk, pv, n, n, 5)
    np.testing.assert_array_equal(o1, o2)


def test_passing_row_order_does_not_matter():
    H, n, hq, hkv, d = 3, 20, 4, 2, 8
    N = H * n
    q, k, v = _rand((N, hq, d), 20), _rand((N, hkv, d), 21), _rand((N, hkv, d), 22)
    idx = compress_indices(_rand((hkv, N), 23), H, n, 6)
    pk, pv = passing_blocks(k, v, idx)
    perm = np.random.default_rng(0).permutation(2 * 6)
    pk2, pv2 = pk.copy(), pv.copy()
    pk2[:, :12], pv2[:, :12] = pk[:, perm], pv[:, perm]
    o1, _, _ = host_attention(q[2 * n:], np.arange(n), 2, k, v, pk, pv, n, 5, 6)
    o2, _, _ = host_attention(q[2 * n:], np.arange(n), 2, k, v, pk2, pv2, n, 5, 6)
    np.testing.assert_allclose(o1, o2, atol=1e-13)


def test_lse_matches_direct_sum():
    n, hq, hkv, d = 30, 2, 1, 4
    q, k, v = _rand((n, hq, d), 24), _rand((n, hkv, d), 25), _rand((n, hkv, d), 26)
    pk = np.zeros((hkv, 0, d))
    rows = np.array([0, 7, 29])
    _, lse, _ = host_attention(q[rows], rows, 0, k, v, pk, pk, n, 0, 0)
    for ri, i in enumerate(rows):
        for j in range(hq):
            direct = math.log(sum(math.exp(float(q[i, j] @ k[c, 0]) / 2.0) for c in range(i + 1)))
            assert abs(lse[ri, j] - direct) < 1e-12


def test_visible_pairs_count():
    # 128K Llama-8B workload: 2,248,212,480 visible pairs per q head
    c = inputs.LLAMA8B_128K
    assert visible_pairs(c.n_hosts, c.block_len, c.anchor_len, c.keep) == 2_248_212_480
    assert visible_pairs(1, 10, 3, 2) == 55


def _visible_mask_count(H, n, A, keep):
    """Brute force: one boolean per (host, local query, key slot), the key
    slots being the A anchor rows, the H*keep rows of the gathered compressed
    blocks and the n rows of the host's own block; each rule of "APB 的主要功能"
    (anchor for hosts >= 1, the blocks of earlier hosts only, local causal
    with the diagonal) is applied slot by slot."""
    total = 0
    for h in range(H):
        for i in range(n):
            mask = np.zeros(A + H * keep + n, dtype=bool)
            for a in range(A):
                mask[a] = h >= 1
            for r in range(H * keep):
                mask[A + r] = (r // keep) < h          # block of host r // keep, before h
            for c in range(n):
                mask[A + H * keep + c] = c <= i
            total += int(mask.sum())
    return total


@pytest.mark.parametrize("H,n,A,keep", [(3, 7, 3, 2), (4, 5, 5, 0), (3, 6, 0, 6), (2, 9, 2, 1)])
def test_visible_pairs_brute_force(H, n, A, keep):
    assert visible_pairs(H, n, A, keep) == _visible_mask_count(H, n, A, keep)


def test_visible_pairs_equals_attended_keys():
    """With q = 0 every visible key gets the same logit, so the oracle's
    attention has exp(lse) = number of keys the row attends; summed over the
    rows of every host this is the visible-pair count of one q head."""
    H, n, A, keep, d = 3, 7, 3, 2, 4
    rng = np.random.default_rng(5)
    k = rng.standard_normal((H * n, 1, d))
    v = rng.standard_normal((H * n, 1, d))
    idx = np.stack([np.stack([np.sort(rng.choice(n, keep, replace=False)) + h * n])
                    for h in range(H)])
    pk, pv = passing_blocks(k, v, idx)
    total = 0.0
    for h in range(H):
        _, lse, _ = host_attention(np.zeros((n, 1, d)), np.arange(n), h, k, v, pk, pv, n, A, keep)
        total += np.exp(lse).sum()
    assert round(total) == visible_pairs(H, n, A, keep) == _visible_mask_count(H, n, A, keep)


# ----------------------------------------------------------------- configs

def test_anchor_fraction_matches_pages():
    g = json.load(open(os.path.join(GOLDEN, "anchor_fraction.json")))
    for cfg in inputs.CONFIGS.values():
        assert cfg.anchor_len / cfg.block_len in g["allowed_fractions"], cfg.name
        assert 0 <= cfg.query_len <= cfg.anchor_len <= cfg.block_len
        assert cfg.n_q_heads % cfg.n_kv_heads == 0


# ----------------------------------------------------------------- query-aware score

def test_query_aware_equals_own_token_score_when_q_is_the_segment():
    # if every token's q equals one fixed row and the segment holds that row,
    # the two readings of the q input coincide
    T, hq, hkv, d = 7, 4, 2, 8
    row = _rand((1, hq, d), 30)
    q = np.repeat(row, T, axis=0)
    k, v = _rand((T, hkv, d), 31), _rand((T, hkv, d), 32)
    w1, b1 = _rand((hkv, 16, 3 * d), 33, 0.1), _rand((hkv, 16), 34, 0.1)
    w2, b2 = _rand((hkv, 16), 35, 0.1), _rand((hkv,), 36, 0.1)
    a = retaining_scores(q, k, v, w1, b1, w2, b2)
    b = retaining_scores_query_aware(np.repeat(row, 3, axis=0), k, v, w1, b1, w2, b2)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)


def test_query_aware_closed_form_and_empty_segment():
    from oracle import retaining_scores_query_aware as qa
    ln3 = math.log(3.0)
    # d = 1, G = 2: segment rows q = (2, 4) and (0, 2) -> mean 2; hidden unit = qseg * ln3/2
    q_seg = np.array([[[2.0], [4.0]], [[0.0], [2.0]]])
    k = np.array([[[5.0]], [[-1.0]]])
    v = np.zeros((2, 1, 1))
    w1 = np.array([[[0.0, 0.0, ln3 / 2], [1.0, 0.0, 0.0]]])   # unit0 = ln3 (qseg), unit1 = k
    b1 = np.zeros((1, 2))
    w2 = np.array([[4.0, 0.0]])
    b2 = np.array([0.5])
    s = qa(q_seg, k, v, w1, b1, w2, b2)
    np.testing.assert_allclose(s[0], [4 * 0.75 * ln3 + 0.5] * 2, atol=1e-14)   # SiLU(ln3) = 3/4 ln3
    # empty segment: q part is zero
    s0 = qa(np.zeros((0, 2, 1)), k, v, w1, b1, w2, b2)
    np.testing.assert_allclose(s0[0], [0.5, 0.5], atol=1e-14)

"""The bench's roofline arithmetic against independent counts (CPU only)."""
import numpy as np

import bench
import oracle
from long_context_sparse_apb_b200 import inputs


def test_visible_pairs_match_the_oracle_count():
    for cfg in (inputs.TINY, inputs.LLAMA8B_32K, inputs.LLAMA8B_128K):
        assert bench.visible_pairs(cfg) == oracle.visible_pairs(cfg.n_hosts, cfg.block_len,
                                                                cfg.anchor_len, cfg.keep)
    assert bench.visible_pairs(inputs.LLAMA8B_128K) == 2_248_212_480
    assert abs(bench.attention_flops(inputs.LLAMA8B_128K, 2_248_212_480) - 36.83e12) < 0.01e12


def test_visited_tiles_follow_the_kernel_grid():
    # one CTA per pair of 128-row query tiles; tile A of CTA u visits
    # na + np + 2u + 1 KV tiles, tile B (when it exists) one more; every
    # visited tile is a full 128 x 128 block of logits
    for cfg in (inputs.TINY, inputs.TINY.replace(n_hosts=5, block_len=300, anchor_len=75,
                                                 keep=130),
                inputs.LLAMA8B_128K):
        n, A, keep, T = cfg.block_len, cfg.anchor_len, cfg.keep, 128
        nq = -(-n // T)
        tot = 0
        for h in range(cfg.n_hosts):
            na = -(-A // T) if (h >= 1 and A > 0) else 0
            np_ = -(-(h * keep) // T)
            for u in range((nq + 1) // 2):
                ta = na + np_ + 2 * u + 1
                tb = ta + 1 if (2 * u + 1) * T < n else 0
                tot += (ta + tb) * T * T
        assert bench.visited_tile_pairs(cfg) == tot
    assert abs(bench.attention_flops(inputs.LLAMA8B_128K,
                                     bench.visited_tile_pairs(inputs.LLAMA8B_128K))
               - 36.97e12) < 0.01e12


def test_compress_bytes():
    # Q once, K and V once, the scores written and read, the indices, and the
    # gather's read and write of K and V rows
    cfg = inputs.LLAMA8B_128K
    N, d, hq, hkv, H, keep = 131072, 128, 32, 8, 8, 2048
    q = N * hq * d * 2
    kv = 2 * N * hkv * d * 2
    scores = 2 * N * hkv * 4
    idx = H * hkv * keep * 4
    gather = 2 * 2 * H * hkv * keep * d * 2
    assert bench.hbm_bytes_compress(cfg) == q + kv + scores + idx + gather == 1_753_743_360


def test_source_rev_ignores_comments_only():
    code = "int f(int x) {\n  return x + 1;\n}\n"
    commented = "// a note\nint f(int x) {  /* why */\n  return x + 1;  // inline\n\n}\n"
    assert bench.source_rev(code) == bench.source_rev(commented)
    assert bench.source_rev(code) != bench.source_rev(code.replace("+ 1", "+ 2"))


def test_kv_head_split_shares_the_work_evenly():
    # the default multi-GPU mode: every rank gets Hkv / N kv heads and their
    # q heads, so the ranks' attention FLOPs and A1-A3 bytes each are 1/N of
    # the sequence's (the per-rank roofline uses the rank's share)
    cfg = inputs.LLAMA8B_128K
    full_fl = bench.attention_flops(cfg, bench.visible_pairs(cfg))
    for world in (1, 2, 4, 8):
        shares = []
        for rank in range(world):
            from long_context_sparse_apb_b200.sharded import kv_head_range
            gb, ge = kv_head_range(cfg.n_kv_heads, rank, world)
            lcfg = cfg.replace(n_q_heads=(ge - gb) * cfg.group, n_kv_heads=ge - gb)
            shares.append(bench.attention_flops(lcfg, bench.visible_pairs(lcfg)))
            assert bench.hbm_bytes_compress(lcfg) * world == bench.hbm_bytes_compress(cfg)
        assert len(set(shares)) == 1 and abs(sum(shares) - full_fl) < 1.0

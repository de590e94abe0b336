"""Workload configurations and seeded synthetic inputs for the APB prefill path.

This module holds sizes and random draws only: no step of the method's own
arithmetic (scoring, selection, gathering, attention) lives here, so both the
CUDA path and the CPU oracle can be fed from it without sharing method code.

The five workloads follow the attention shapes the APB pages name for their
backbones (Llama-3.1-8B, Qwen-2.5-14B, Llama-3-8B-1M; "APB: Accelerating
Distributed Long-Context Inference by Passing Compressed Context Blocks across
GPUs", the juejin.cn post, section "如何运行 APB", retaining-head table) at the
32K-512K context lengths the pages' long-context benchmarks use.  The pages'
datasets (RULER, InfiniteBench, LongBench, NIAH) are not reproduced: seeded
Gaussian Q/K/V with RoPE structure and planted "needle" keys stand in for them.

Recipe (all draws on CPU torch generators, one generator per stream):
  * Q, K, V: for tensor id T in (Q=1, K=2, V=3) and host h, a generator seeded
    with ``mix(seed, T, h)`` draws the host's block of n rows, shape
    [n, heads, d], N(0, 1) (V of the Qwen workload: std 0.5).
  * RoPE (rotate-half, inv_freq = theta^(-2i/d), position = global token
    index, angles in fp64) is applied to Q and K in fp32 where a theta is given.
  * Needles: per host, ``needles_per_host`` positions drawn without
    replacement (generator ``mix(seed, 200, h)``) from the host's block minus
    the anchor rows [0, A); for every kv head g the key row is set to
    3*sqrt(d)*u_g, u_g the unit vector of the mean of post-RoPE Q over the
    query segment [0, q_len) and the q heads of group g.  V is unchanged.
  * Then Q, K, V are rounded to bf16 (round-to-nearest-even).
  * Retaining-head stand-in weights (generator ``mix(seed, 100, 0)``), fp32
    N(0, 0.02), drawn in order W1 [Hkv, hidden, 3d], b1 [Hkv, hidden],
    w2 [Hkv, hidden], b2 [Hkv].
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class APBConfig:
    name: str
    n_hosts: int          # H: virtual hosts (context blocks)
    block_len: int        # n: tokens per host
    anchor_len: int       # A: anchor rows [0, A), visible to hosts >= 1
    query_len: int        # q_len: query segment at the start of the anchor
    keep: int             # top-k per (host, kv head)
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    mlp_hidden: int = 256
    seed: int = 0
    rope_theta: Optional[float] = None
    v_std: float = 1.0
    needles_per_host: int = 0
    # rows per host that full-size parity checks against the oracle (None = all)
    sample_rows_per_host: Optional[int] = None

    @property
    def seq_len(self) -> int:
        return self.n_hosts * self.block_len

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def replace(self, **kw) -> "APBConfig":
        return dataclasses.replace(self, **kw)


# The five workloads (attention shapes of the pages' backbones; see module doc).
TINY = APBConfig("tiny_2k", n_hosts=4, block_len=512, anchor_len=128, query_len=32,
                 keep=64, n_q_heads=4, n_kv_heads=2, head_dim=64, seed=0,
                 rope_theta=None, needles_per_host=4)
LLAMA8B_32K = APBConfig("llama8b_32k", n_hosts=8, block_len=4096, anchor_len=1024,
                        query_len=64, keep=512, n_q_heads=32, n_kv_heads=8,
                        head_dim=128, seed=1, rope_theta=5e5, needles_per_host=16)
LLAMA8B_128K = APBConfig("llama8b_128k", n_hosts=8, block_len=16384, anchor_len=2048,
                         query_len=128, keep=2048, n_q_heads=32, n_kv_heads=8,
                         head_dim=128, seed=2, rope_theta=5e5, needles_per_host=32)
QWEN14B_128K = APBConfig("qwen14b_128k", n_hosts=8, block_len=16384, anchor_len=4096,
                         query_len=128, keep=1024, n_q_heads=40, n_kv_heads=8,
                         head_dim=128, seed=3, rope_theta=1e6, v_std=0.5,
                         needles_per_host=0)
LLAMA8B_1M_512K = APBConfig("llama8b_1m_512k", n_hosts=16, block_len=32768,
                            anchor_len=4096, query_len=256, keep=2048, n_q_heads=32,
                            n_kv_heads=8, head_dim=128, seed=4, rope_theta=None,
                            needles_per_host=64, sample_rows_per_host=4096)

CONFIGS: Dict[str, APBConfig] = {c.name: c for c in
                                 (TINY, LLAMA8B_32K, LLAMA8B_128K, QWEN14B_128K,
                                  LLAMA8B_1M_512K)}

_TID_Q, _TID_K, _TID_V, _TID_W, _TID_NEEDLE = 1, 2, 3, 100, 200


def mix(seed: int, tensor_id: int, index: int) -> int:
    """Deterministic generator seed for one stream (tensor, host)."""
    return (seed * 1_000_003 + tensor_id * 10_007 + index) % (2 ** 62)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _rope_(x: torch.Tensor, pos0: int, theta: float) -> None:
    """In-place rotate-half RoPE on x [n, heads, d] (fp32), positions pos0.."""
    n, _, d = x.shape
    half = d // 2
    inv = theta ** (-torch.arange(0, half, dtype=torch.float64) * 2.0 / d)
    ang = torch.arange(pos0, pos0 + n, dtype=torch.float64)[:, None] * inv[None, :]
    cos = ang.cos().to(torch.float32)[:, None, :]
    sin = ang.sin().to(torch.float32)[:, None, :]
    x1 = x[..., :half].clone()
    x2 = x[..., half:].clone()
    x[..., :half] = x1 * cos - x2 * sin
    x[..., half:] = x2 * cos + x1 * sin


def needle_positions(cfg: APBConfig, host: int) -> torch.Tensor:
    """Global positions of the planted needle keys of one host (sorted)."""
    n, a = cfg.block_len, cfg.anchor_len
    lo = max(host * n, a)
    hi = host * n + n
    m = min(cfg.needles_per_host, max(hi - lo, 0))
    if m == 0:
        return torch.zeros(0, dtype=torch.int64)
    perm = torch.randperm(hi - lo, generator=_gen(mix(cfg.seed, _TID_NEEDLE, host)))
    return torch.sort(perm[:m] + lo).values


def generate_weights(cfg: APBConfig) -> Dict[str, torch.Tensor]:
    g = _gen(mix(cfg.seed, _TID_W, 0))
    hkv, hid, d = cfg.n_kv_heads, cfg.mlp_hidden, cfg.head_dim
    w1 = torch.randn((hkv, hid, 3 * d), generator=g) * 0.02
    b1 = torch.randn((hkv, hid), generator=g) * 0.02
    w2 = torch.randn((hkv, hid), generator=g) * 0.02
    b2 = torch.randn((hkv,), generator=g) * 0.02
    return {"w1": w1.contiguous(), "b1": b1.contiguous(),
            "w2": w2.contiguous(), "b2": b2.contiguous()}


def _q_block(cfg: APBConfig, h: int) -> torch.Tensor:
    """Host h's post-RoPE fp32 Q block [n, Hq, d]."""
    n, d = cfg.block_len, cfg.head_dim
    x = torch.randn((n, cfg.n_q_heads, d), generator=_gen(mix(cfg.seed, _TID_Q, h)))
    if cfg.rope_theta is not None:
        _rope_(x, h * n, cfg.rope_theta)
    return x


def _qseg_mean(cfg: APBConfig, q0: torch.Tensor) -> torch.Tensor:
    """[Hkv, d] mean of post-RoPE fp32 Q over the query segment and the group."""
    hkv, G, d = cfg.n_kv_heads, cfg.group, cfg.head_dim
    if cfg.query_len == 0:
        return torch.zeros(hkv, d)
    return q0[: cfg.query_len].reshape(cfg.query_len, hkv, G, d).mean(dim=(0, 2))


def _kv_block(cfg: APBConfig, h: int, qseg_mean: torch.Tensor, which: int) -> torch.Tensor:
    """Host h's K (which = K id, needles planted) or V block, fp32."""
    n, d, hkv = cfg.block_len, cfg.head_dim, cfg.n_kv_heads
    x = torch.randn((n, hkv, d), generator=_gen(mix(cfg.seed, which, h)))
    if which == _TID_K:
        if cfg.rope_theta is not None:
            _rope_(x, h * n, cfg.rope_theta)
        pos = needle_positions(cfg, h)
        if pos.numel():
            u = qseg_mean / qseg_mean.norm(dim=-1, keepdim=True).clamp_min(1e-30)
            x[pos - h * n] = (3.0 * math.sqrt(d) * u)[None, :, :]
    elif cfg.v_std != 1.0:
        x *= cfg.v_std
    return x


def generate(cfg: APBConfig) -> Dict[str, torch.Tensor]:
    """All inputs of one workload as CPU tensors.

    Returns q [N, Hq, d], k [N, Hkv, d], v [N, Hkv, d] (bf16, token-major),
    w1/b1/w2/b2 (fp32) and ``needles`` (int64 global positions).
    """
    H, n, d = cfg.n_hosts, cfg.block_len, cfg.head_dim
    hq, hkv = cfg.n_q_heads, cfg.n_kv_heads
    N = H * n
    q = torch.empty((N, hq, d), dtype=torch.bfloat16)
    k = torch.empty((N, hkv, d), dtype=torch.bfloat16)
    v = torch.empty((N, hkv, d), dtype=torch.bfloat16)
    qseg_mean = None
    for h in range(H):
        x = _q_block(cfg, h)
        if h == 0:
            qseg_mean = _qseg_mean(cfg, x)
        q[h * n:(h + 1) * n] = x.to(torch.bfloat16)
    for h in range(H):
        k[h * n:(h + 1) * n] = _kv_block(cfg, h, qseg_mean, _TID_K).to(torch.bfloat16)
    for h in range(H):
        v[h * n:(h + 1) * n] = _kv_block(cfg, h, qseg_mean, _TID_V).to(torch.bfloat16)

    out = {"q": q, "k": k, "v": v}
    out.update(generate_weights(cfg))
    out["needles"] = torch.cat([needle_positions(cfg, h) for h in range(H)])
    return out


def generate_local(cfg: APBConfig, host_begin: int, host_end: int,
                   host_stride: int = 1) -> Dict[str, torch.Tensor]:
    """What one GPU of a host-sharded prefill holds: q of the hosts
    range(host_begin, host_end, host_stride) and k/v with the anchor's rows
    [0, A) first, then those hosts' rows, in that order (each host prepends
    the anchor to its block).  Values equal the matching rows of
    generate(cfg)."""
    n, A = cfg.block_len, cfg.anchor_len
    q0 = _q_block(cfg, 0)
    qseg_mean = _qseg_mean(cfg, q0)
    hosts = range(host_begin, host_end, host_stride)
    q = torch.cat([(q0 if h == 0 else _q_block(cfg, h)).to(torch.bfloat16) for h in hosts])
    out = {"q": q}
    for name, tid in (("k", _TID_K), ("v", _TID_V)):
        anchor = _kv_block(cfg, 0, qseg_mean, tid)[:A].to(torch.bfloat16)
        blocks = [_kv_block(cfg, h, qseg_mean, tid).to(torch.bfloat16) for h in hosts]
        out[name] = torch.cat([anchor] + blocks)
    out.update(generate_weights(cfg))
    return out


def sample_rows(cfg: APBConfig, host: int, count: int) -> torch.Tensor:
    """Seeded sample of local query rows of one host, always holding the
    block's first and last rows, the anchor's last row and the rows on each
    side of the first 128-row tile boundary (when in range)."""
    n = cfg.block_len
    must = {0, n - 1, 127, 128, cfg.anchor_len - 1}
    must = sorted(r for r in must if 0 <= r < n)
    if count >= n:
        return torch.arange(n, dtype=torch.int64)
    g = _gen(cfg.seed + 1000 * host)
    perm = torch.randperm(n, generator=g)
    chosen = list(dict.fromkeys(must + perm.tolist()))[:max(count, len(must))]
    return torch.sort(torch.tensor(chosen, dtype=torch.int64)).values

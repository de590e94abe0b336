"""APB prefill with the hosts spread over several GPUs: the distributed form
the pages describe ("APB 的主要功能": the sequence is split evenly over hosts,
each host prepends the anchor block to its context block, compresses its KV
with the retaining heads, the compressed blocks are all-gathered, and each host
attends over anchor + passing block + its own block).

One process per GPU; rank r owns the contiguous hosts [r*H/W, (r+1)*H/W).
Per step, on each rank:
  1. for every owned host: score + top-k (apb_score_compress on that host's
     block) and its compressed block, written straight into the host's rows
     [h*keep, (h+1)*keep) of a full token-major passing buffer
     (apb_build_passing);
  2. one all-gather of the passing buffer's K rows and one of its V rows
     (each rank contributes its contiguous chunk; the result is all hosts'
     blocks in host order, because ranks own hosts in order);
  3. attention of the owned hosts on the rank-local buffers
     (apb_block_attention_hosts).
Every step of the data path runs in the library's kernels; the exchange is
the collective passed in (NCCL all_gather_into_tensor between GPUs).
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch

from . import _lib as apb


def host_range(n_hosts: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous hosts owned by `rank` (n_hosts must divide evenly)."""
    if n_hosts % world != 0:
        raise ValueError(f"{n_hosts} hosts do not split evenly over {world} ranks")
    per = n_hosts // world
    return rank * per, (rank + 1) * per


def kv_head_range(n_kv_heads: int, rank: int, world: int) -> Tuple[int, int]:
    """Kv heads owned by `rank` in the kv-head partitioning (the other natural
    split of this path: every (host, kv head) unit is independent, so each
    GPU runs the whole path on its kv heads and their q heads, with no
    collective at all)."""
    if n_kv_heads % world != 0:
        raise ValueError(f"{n_kv_heads} kv heads do not split evenly over {world} ranks")
    per = n_kv_heads // world
    return rank * per, (rank + 1) * per


def head_slice(x: dict, n_q_heads: int, n_kv_heads: int, gb: int, ge: int) -> dict:
    """The inputs of kv heads [gb, ge) and their q heads, contiguous."""
    G = n_q_heads // n_kv_heads
    out = {"q": x["q"][:, gb * G:ge * G].contiguous(), "k": x["k"][:, gb:ge].contiguous(),
           "v": x["v"][:, gb:ge].contiguous()}
    for w in ("w1", "b1", "w2", "b2"):
        out[w] = x[w][gb:ge].contiguous()
    return out


def nccl_all_gather(group=None) -> Callable[[torch.Tensor, torch.Tensor], None]:
    """In-place all-gather of a rank's chunk into the full buffer (NCCL):
    `chunk` must be this rank's slice of `full`."""
    import torch.distributed as dist

    def gather(full: torch.Tensor, chunk: torch.Tensor) -> None:
        dist.all_gather_into_tensor(full, chunk, group=group)
    return gather


def list_all_gather(group=None) -> Callable[[torch.Tensor, torch.Tensor], None]:
    """The same exchange through torch.distributed.all_gather (any backend,
    used by the CPU tests with gloo)."""
    import torch.distributed as dist

    def gather(full: torch.Tensor, chunk: torch.Tensor) -> None:
        world = dist.get_world_size(group)
        parts = list(full.chunk(world, dim=0))
        dist.all_gather(parts, chunk.clone(), group=group)
    return gather


class ShardedPrefill:
    """One rank's share of a host-sharded prefill of one sequence.

    c: the whole sequence's apb_config.  all_gather(full, chunk) fills `full`
    with every rank's chunk in rank order (None: the caller places the other
    ranks' chunks itself, e.g. when several ranks share one GPU in a test).
    """

    def __init__(self, c: apb.Config, rank: int, world: int, device="cuda",
                 all_gather: Optional[Callable] = None):
        self.c = c
        self.rank, self.world = rank, world
        self.hb, self.he = host_range(c.n_hosts, rank, world)
        self.all_gather = all_gather
        n, keep, hkv, d = c.block_len, c.keep, c.n_kv_heads, c.head_dim
        # single-host config for the per-host compression calls
        self.c1 = apb.make_config(None, n_hosts=1, block_len=n, anchor_len=c.anchor_len,
                                  query_len=c.query_len, keep=keep, n_q_heads=c.n_q_heads,
                                  n_kv_heads=hkv, head_dim=d, mlp_hidden=c.mlp_hidden,
                                  softmax_scale=c.softmax_scale)
        dev = torch.device(device)
        self.workspace = apb.new_workspace(self.c1, dev)
        self.idx = torch.empty((self.he - self.hb, 1, hkv, keep), dtype=torch.int32, device=dev)
        shape = (c.n_hosts * keep, hkv, d)
        self.pass_k = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        self.pass_v = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        self.out = torch.empty(((self.he - self.hb) * n, c.n_q_heads, d), dtype=torch.bfloat16,
                               device=dev)

    def compress(self, q, kv_k, kv_v, w1, b1, w2, b2, stream=None, query_aware=False):
        """Steps 1: compressed blocks of the owned hosts into their rows."""
        n, A, keep = self.c.block_len, self.c.anchor_len, self.c.keep
        for i, h in enumerate(range(self.hb, self.he)):
            qs = q[i * n:(i + 1) * n]
            ks = kv_k[A + i * n:A + (i + 1) * n]
            vs = kv_v[A + i * n:A + (i + 1) * n]
            apb.score_compress(self.c1, qs, ks, vs, w1, b1, w2, b2, idx=self.idx[i],
                               workspace=self.workspace, stream=stream, query_aware=query_aware)
            if keep > 0:
                apb.build_passing(self.c1, ks, vs, self.idx[i],
                                  self.pass_k[h * keep:(h + 1) * keep],
                                  self.pass_v[h * keep:(h + 1) * keep], stream=stream)

    def exchange(self):
        """Step 2: all ranks' compressed blocks into every rank's buffer."""
        keep = self.c.keep
        if self.all_gather is None or keep == 0 or self.world == 1:
            return
        rows = slice(self.hb * keep, self.he * keep)
        self.all_gather(self.pass_k, self.pass_k[rows])
        self.all_gather(self.pass_v, self.pass_v[rows])

    def attend(self, q, kv_k, kv_v, stream=None, lse=None):
        """Step 3: attention of the owned hosts."""
        out, _ = apb.block_attention_hosts(self.c, self.hb, self.he, q, kv_k, kv_v, self.pass_k,
                                           self.pass_v, out=self.out, lse=lse,
                                           workspace=self.workspace, stream=stream)
        return out

    def __call__(self, q, kv_k, kv_v, w1, b1, w2, b2, stream=None):
        self.compress(q, kv_k, kv_v, w1, b1, w2, b2, stream=stream)
        self.exchange()
        return self.attend(q, kv_k, kv_v, stream=stream)

"""APB prefill with the hosts spread over several GPUs: the distributed form
the pages describe ("APB 的主要功能": the sequence is split evenly over hosts,
each host prepends the anchor block to its context block, compresses its KV
with the retaining heads, the compressed blocks are all-gathered, and each host
attends over anchor + passing block + its own block).

One process per GPU.  Rank r of W owns H/W hosts, either round-robin (hosts
r, r+W, r+2W, ...: the default, which balances the work, since a host's
attention grows with its index through the passing block) or contiguous
(hosts [r*H/W, (r+1)*H/W)).  Per step, on each rank:
  1. for every owned host: score + top-k and its compressed block, written
     straight into the host's rows [h*keep, (h+1)*keep) of a full token-major
     passing buffer (apb_score_compress_pass: the gather runs in the top-k
     launch; the query-aware variant takes apb_score_compress_query_aware +
     apb_build_passing);
  2. all-gathers of the passing buffer's K and V rows that leave every
     host's block in host order: round-robin, one per round i over the rows
     of hosts [i*W, (i+1)*W) (rank r contributes host i*W + r); contiguous,
     one over the whole buffer (rank r contributes its hosts' chunk);
  3. attention of the owned hosts on the rank-local buffers
     (apb_block_attention_host_set).
Every step of the data path runs in the library's kernels; the exchange is
the collective passed in (NCCL all_gather_into_tensor between GPUs).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple

import torch

from . import _lib as apb


def host_range(n_hosts: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous hosts owned by `rank` (n_hosts must divide evenly)."""
    if n_hosts % world != 0:
        raise ValueError(f"{n_hosts} hosts do not split evenly over {world} ranks")
    per = n_hosts // world
    return rank * per, (rank + 1) * per


def host_set(n_hosts: int, rank: int, world: int, order: str = "round_robin") -> Tuple[int, int, int]:
    """(first, count, stride) of the hosts owned by `rank`: round_robin owns
    rank, rank+W, ...; contiguous owns [rank*H/W, (rank+1)*H/W)."""
    first, end = host_range(n_hosts, rank, world)
    if order == "contiguous":
        return first, end - first, 1
    if order == "round_robin":
        return rank, end - first, world
    raise ValueError(f"unknown host order {order!r}")


def exchange_chunks(n_hosts: int, keep: int, rank: int, world: int,
                    order: str = "round_robin") -> List[Tuple[slice, slice]]:
    """Row ranges (full, chunk) of the passing buffer for the all-gathers of
    the exchange: after all_gather(full, chunk) for each pair (every rank
    passing its own chunk, which lies inside full at position `rank`), the
    buffer holds every host's block in host order."""
    first, count, stride = host_set(n_hosts, rank, world, order)
    if order == "contiguous":
        return [(slice(0, n_hosts * keep), slice(first * keep, (first + count) * keep))]
    W = world
    return [(slice(i * W * keep, (i + 1) * W * keep),
             slice((i * W + rank) * keep, (i * W + rank + 1) * keep)) for i in range(count)]


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


def tensor_all_gather(group=None) -> Callable[[torch.Tensor, torch.Tensor], None]:
    """In-place all-gather of a rank's chunk into the full buffer through
    torch.distributed.all_gather_into_tensor: NCCL between GPUs, gloo between
    CPU ranks.  `chunk` must be this rank's slot of `full` (slot `rank` of
    `world` equal parts)."""
    import torch.distributed as dist

    def gather(full: torch.Tensor, chunk: torch.Tensor) -> None:
        dist.all_gather_into_tensor(full, chunk, group=group)
    return gather


class ShardedPrefill:
    """One rank's share of a host-sharded prefill of one sequence.

    c: the whole sequence's apb_config.  all_gather(full, chunk) fills `full`
    with every rank's chunk in rank order (None: the caller places the other
    ranks' chunks itself, e.g. when several ranks share one GPU in a test).
    """

    def __init__(self, c: apb.Config, rank: int, world: int, device="cuda",
                 all_gather: Optional[Callable] = None, order: str = "round_robin"):
        self.c = c
        self.rank, self.world = rank, world
        self.order = order
        self.first, self.count, self.stride = host_set(c.n_hosts, rank, world, order)
        self.hosts = [self.first + i * self.stride for i in range(self.count)]
        self.all_gather = all_gather
        n, keep, hkv, d = c.block_len, c.keep, c.n_kv_heads, c.head_dim
        # single-host config for the per-host compression calls
        self.c1 = apb.make_config(None, n_hosts=1, block_len=n, anchor_len=c.anchor_len,
                                  query_len=c.query_len, keep=keep, n_q_heads=c.n_q_heads,
                                  n_kv_heads=hkv, head_dim=d, mlp_hidden=c.mlp_hidden,
                                  softmax_scale=c.softmax_scale)
        dev = torch.device(device)
        self.workspace = apb.new_workspace(self.c1, dev)
        self.idx = torch.empty((self.count, 1, hkv, keep), dtype=torch.int32, device=dev)
        shape = (c.n_hosts * keep, hkv, d)
        self.pass_k = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        self.pass_v = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        self.out = torch.empty((self.count * n, c.n_q_heads, d), dtype=torch.bfloat16,
                               device=dev)

    def compress(self, q, kv_k, kv_v, w1, b1, w2, b2, stream=None, query_aware=False):
        """Steps 1: compressed blocks of the owned hosts into their rows."""
        n, A, keep = self.c.block_len, self.c.anchor_len, self.c.keep
        for i, h in enumerate(self.hosts):
            qs = q[i * n:(i + 1) * n]
            ks = kv_k[A + i * n:A + (i + 1) * n]
            vs = kv_v[A + i * n:A + (i + 1) * n]
            if keep > 0 and not query_aware:
                apb.score_compress_pass(self.c1, qs, ks, vs, w1, b1, w2, b2,
                                        self.pass_k[h * keep:(h + 1) * keep],
                                        self.pass_v[h * keep:(h + 1) * keep], idx=self.idx[i],
                                        workspace=self.workspace, stream=stream)
                continue
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
        for full, chunk in exchange_chunks(self.c.n_hosts, keep, self.rank, self.world,
                                           self.order):
            self.all_gather(self.pass_k[full], self.pass_k[chunk])
            self.all_gather(self.pass_v[full], self.pass_v[chunk])

    def attend(self, q, kv_k, kv_v, stream=None, lse=None):
        """Step 3: attention of the owned hosts."""
        out, _ = apb.block_attention_host_set(self.c, self.first, self.count, self.stride, q, kv_k,
                                              kv_v, self.pass_k, self.pass_v, out=self.out,
                                              lse=lse, workspace=self.workspace, stream=stream)
        return out

    def __call__(self, q, kv_k, kv_v, w1, b1, w2, b2, stream=None):
        self.compress(q, kv_k, kv_v, w1, b1, w2, b2, stream=stream)
        self.exchange()
        return self.attend(q, kv_k, kv_v, stream=stream)

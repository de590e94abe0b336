"""CPU oracle of the APB per-host prefill path (NumPy, float64).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
executes this module: only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may.  It shares no code with the CUDA library
and imports nothing from the package; inputs arrive as plain arrays.

Source of the method: "APB: Accelerating Distributed Long-Context Inference by
Passing Compressed Context Blocks across GPUs" (arXiv 2502.12085), as described
on the juejin.cn post about APB, sections "APB 的主要功能" (main features) and
"APB 的技术原理" (technical principles):

  * the input is split evenly into H context blocks, one per host;
  * every host's local block is preceded by an anchor block, the start of the
    input sequence, 1/4 or 1/8 of a block long, with the query embedded at its
    start;
  * each host compresses its KV with retaining heads (Locret) and keeps the
    important KV pairs; the compressed blocks are all-gathered and each host
    builds a passing block from the compressed blocks of the hosts before it;
  * attention on each host runs over anchor + passing + local block, and the
    passing block is discarded afterwards.

Readings taken where the pages are silent:
  R1  host 0 has no anchor (its block already starts the sequence);
  R2  the anchor is rows [0, A) of K/V; the query segment is rows [0, q_len);
  R3  anchor and passing are attended in full, the local block causally with
      the diagonal included; softmax scale 1/sqrt(d) unless given;
  R4  a token of host 0 chosen by top-k may appear both in the anchor and in
      a later host's passing block; it is kept twice;
  R5  the retaining-head stand-in scores token t for kv head g from
      concat(k[t,g], v[t,g], mean over the group's q heads of q[t,j]) through
      Linear(3d, hidden) -> SiLU -> Linear(hidden, 1);
  R6  q head j uses kv head j // G (consecutive grouping);
  R5b (query-aware variant) the q part of the MLP input is the mean of the
      query segment over its rows and the group's q heads, for every token;
  R7  top-k ties: the lower position wins; indices are returned ascending.

Every function below is checked by ``tests/test_oracle_pins.py`` against
closed forms, brute force and library routines (dense causal attention).
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def _f64(x):
    return np.asarray(x, dtype=F64)


def retaining_scores(q, k, v, w1, b1, w2, b2):
    """Retaining-head stand-in score of every token for every kv head.

    Follows "APB 的主要功能" (KV compression with Locret's retaining heads) with
    the stand-in MLP of reading R5: for token t and kv head g,
        x = [k[t,g] ; v[t,g] ; (1/G) * sum_{j: j//G == g} q[t,j]]   (3d)
        s[g,t] = w2[g] . SiLU(W1[g] x + b1[g]) + b2[g],  SiLU(z) = z/(1+e^-z).

    q [T, Hq, d], k/v [T, Hkv, d] (any float dtype; upcast exactly),
    w1 [Hkv, hidden, 3d], b1 [Hkv, hidden], w2 [Hkv, hidden], b2 [Hkv].
    Returns s [Hkv, T] float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    w1, b1, w2, b2 = _f64(w1), _f64(b1), _f64(w2), _f64(b2)
    T, hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    qbar = q.reshape(T, hkv, G, d).mean(axis=2)          # [T, Hkv, d]
    s = np.empty((hkv, T), dtype=F64)
    with np.errstate(over="ignore"):
        for g in range(hkv):
            x = np.concatenate([k[:, g, :], v[:, g, :], qbar[:, g, :]], axis=1)
            z = x @ w1[g].T + b1[g]                        # [T, hidden]
            a = z / (1.0 + np.exp(-z))
            s[g] = a @ w2[g] + b2[g]
    return s


def retaining_scores_query_aware(q_seg, k, v, w1, b1, w2, b2):
    """Query-aware variant of the stand-in score ("APB 的技术原理": the query is
    embedded at the start of the anchor so that the compressor sees it).

    Reading R5b: the q part of the MLP input is the mean of the query segment
    (rows [0, q_len) of the sequence) over its rows and over the group's q
    heads, the same for every token:
        qseg[g] = mean_{r < q_len, j: j//G == g} q[r, j]     (0 if q_len == 0)
        x = [k[t,g] ; v[t,g] ; qseg[g]],   s[g,t] as in retaining_scores.

    q_seg [q_len, Hq, d] (the query segment), k/v [T, Hkv, d], weights as in
    retaining_scores.  Returns s [Hkv, T] float64.
    """
    q_seg, k, v = _f64(q_seg), _f64(k), _f64(v)
    w1, b1, w2, b2 = _f64(w1), _f64(b1), _f64(w2), _f64(b2)
    T, hkv, d = k.shape
    L, hq, _ = q_seg.shape
    G = hq // hkv
    if L > 0:
        qm = q_seg.reshape(L, hkv, G, d).mean(axis=(0, 2))   # [Hkv, d]
    else:
        qm = np.zeros((hkv, d))
    s = np.empty((hkv, T), dtype=F64)
    with np.errstate(over="ignore"):
        for g in range(hkv):
            x = np.concatenate([k[:, g, :], v[:, g, :], np.broadcast_to(qm[g], (T, d))], axis=1)
            z = x @ w1[g].T + b1[g]
            a = z / (1.0 + np.exp(-z))
            s[g] = a @ w2[g] + b2[g]
    return s


def compress_indices(s, n_hosts, block_len, keep):
    """Top-`keep` tokens of every (host, kv head): the host's compressed block.

    "APB 的技术原理": each context block is compressed to its important KV pairs
    before being communicated.  Selection by score, ties to the lower position
    (R7), result as global positions in ascending order.

    s [Hkv, N] -> idx [H, Hkv, keep] int64.
    """
    s = _f64(s)
    hkv = s.shape[0]
    n = block_len
    idx = np.empty((n_hosts, hkv, keep), dtype=np.int64)
    for h in range(n_hosts):
        for g in range(hkv):
            seg = s[g, h * n:(h + 1) * n]
            order = np.argsort(-seg, kind="stable")[:keep]   # stable: lower index first on ties
            idx[h, g] = np.sort(order) + h * n
    return idx


def passing_blocks(k, v, idx):
    """All-gathered compressed blocks laid out in host order.

    "APB 的主要功能" (communication): the compressed blocks are all-gathered and
    host h's passing block is built from the blocks of the hosts before it.
    Row h'*keep + r of kv head g holds token idx[h', g, r]; host h's passing
    block is therefore rows [0, h*keep) of this layout.

    k, v [N, Hkv, d]; idx [H, Hkv, keep] -> pass_k, pass_v [Hkv, H*keep, d]
    (same dtype as k/v, values copied exactly).
    """
    k = np.asarray(k)
    v = np.asarray(v)
    H, hkv, keep = idx.shape
    d = k.shape[2]
    pk = np.empty((hkv, H * keep, d), dtype=k.dtype)
    pv = np.empty((hkv, H * keep, d), dtype=v.dtype)
    for g in range(hkv):
        rows = idx[:, g, :].reshape(-1)
        pk[g] = k[rows, g, :]
        pv[g] = v[rows, g, :]
    return pk, pv


def host_attention(q_rows, rows, host, k, v, pass_k, pass_v, block_len,
                   anchor_len, keep, scale=None, heads=None, chunk=256):
    """Attention of some local queries of one host over anchor+passing+local.

    "APB 的主要功能" (computation): each host attends over the anchor block,
    the passing block and its local context block; readings R1-R3, R6.
    For local query i (global t = host*n + i) and q head j, g = j // G:
        keys  = K[0:A, g] (host >= 1 only)  ++  pass_k[g, 0:host*keep]
                ++ K[host*n : host*n + i + 1, g]
        o     = softmax(q . keys^T * scale) @ values.

    q_rows [R, Hq, d] are the queries at local rows `rows` [R]; k, v [N, Hkv, d]
    are the full key/value arrays; pass_k/pass_v [Hkv, H*keep, d].
    `heads` restricts the q heads computed (default all).
    Returns (o [R, nh, d], lse [R, nh], rowsum [R, nh]) in float64, where
    lse is the natural log-sum-exp of the scaled logits and rowsum the sum of
    the softmax probabilities (1 up to rounding).
    """
    q_rows = _f64(q_rows)
    rows = np.asarray(rows, dtype=np.int64)
    R, hq, d = q_rows.shape
    hkv = k.shape[1]
    G = hq // hkv
    n = block_len
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    heads = list(range(hq)) if heads is None else list(heads)
    A = anchor_len if host >= 1 else 0                    # R1
    P = host * keep
    o = np.zeros((R, len(heads), d), dtype=F64)
    lse = np.zeros((R, len(heads)), dtype=F64)
    rowsum = np.zeros((R, len(heads)), dtype=F64)
    if R == 0:
        return o, lse, rowsum
    for hi, j in enumerate(heads):
        g = j // G                                          # R6
        for c0 in range(0, R, chunk):
            rr = rows[c0:c0 + chunk]
            last = int(rr.max())
            kk = np.concatenate([_f64(k[0:A, g]), _f64(pass_k[g, 0:P]),
                                 _f64(k[host * n: host * n + last + 1, g])], axis=0)
            vv = np.concatenate([_f64(v[0:A, g]), _f64(pass_v[g, 0:P]),
                                 _f64(v[host * n: host * n + last + 1, g])], axis=0)
            logits = (q_rows[c0:c0 + chunk, j, :] @ kk.T) * scale
            # causal mask on the local part: local key c visible iff c <= i
            loc = np.arange(last + 1)[None, :]
            hidden = loc > rr[:, None]
            logits[:, A + P:][hidden] = -np.inf
            m = logits.max(axis=1, keepdims=True)
            p = np.exp(logits - m)
            l = p.sum(axis=1, keepdims=True)
            prob = p / l
            o[c0:c0 + chunk, hi] = prob @ vv
            lse[c0:c0 + chunk, hi] = (m + np.log(l))[:, 0]
            rowsum[c0:c0 + chunk, hi] = prob.sum(axis=1)
    return o, lse, rowsum


def visible_pairs(n_hosts, block_len, anchor_len, keep):
    """Number of (query, key) pairs one q head attends over the whole sequence:
    sum over hosts of n(n+1)/2 causal pairs, n*A anchor pairs (hosts >= 1) and
    n*h*keep passing pairs."""
    n = block_len
    tot = 0
    for h in range(n_hosts):
        tot += n * (n + 1) // 2 + (n * anchor_len if h >= 1 else 0) + n * h * keep
    return tot

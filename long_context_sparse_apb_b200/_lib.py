"""Python binding of the C ABI in include/apb.h (argument marshalling only).

Every step of the path runs in the CUDA kernels of ``libapb.so``; this module
checks tensor devices, dtypes and shapes, allocates outputs with torch when
the caller gives none, and passes raw device pointers plus the current torch
stream.  Importing it fails loudly when the in-tree library is missing.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libapb.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "apb.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m long_context_sparse_apb_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

APB_OK, APB_ERR_INVALID_ARG, APB_ERR_UNSUPPORTED, APB_ERR_CUDA, APB_ERR_TIMEOUT = range(5)


class Config(ctypes.Structure):
    _fields_ = [("n_hosts", ctypes.c_int32), ("block_len", ctypes.c_int32),
                ("anchor_len", ctypes.c_int32), ("query_len", ctypes.c_int32),
                ("keep", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("mlp_hidden", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]


_P = ctypes.c_void_p
_lib.apb_workspace_bytes.argtypes = [ctypes.POINTER(Config)]
_lib.apb_workspace_bytes.restype = ctypes.c_size_t
_lib.apb_score_compress.argtypes = [ctypes.POINTER(Config)] + [_P] * 10 + [ctypes.c_size_t, _P]
_lib.apb_score_compress.restype = ctypes.c_int
_lib.apb_score_compress_query_aware.argtypes = _lib.apb_score_compress.argtypes
_lib.apb_score_compress_query_aware.restype = ctypes.c_int
_lib.apb_score_compress_pass.argtypes = [ctypes.POINTER(Config)] + [_P] * 12 + [ctypes.c_size_t, _P]
_lib.apb_score_compress_pass.restype = ctypes.c_int
_lib.apb_prefill_workspace_bytes.argtypes = [ctypes.POINTER(Config)]
_lib.apb_prefill_workspace_bytes.restype = ctypes.c_size_t
_lib.apb_prefill.argtypes = [ctypes.POINTER(Config)] + [_P] * 10 + [ctypes.c_size_t, _P]
_lib.apb_prefill.restype = ctypes.c_int
_lib.apb_build_passing.argtypes = [ctypes.POINTER(Config)] + [_P] * 6
_lib.apb_build_passing.restype = ctypes.c_int
_lib.apb_block_attention.argtypes = [ctypes.POINTER(Config)] + [_P] * 8 + [ctypes.c_size_t, _P]
_lib.apb_block_attention.restype = ctypes.c_int
_lib.apb_block_attention_hosts.argtypes = ([ctypes.POINTER(Config), ctypes.c_int32, ctypes.c_int32]
                                           + [_P] * 8 + [ctypes.c_size_t, _P])
_lib.apb_block_attention_hosts.restype = ctypes.c_int
_lib.apb_block_attention_range.argtypes = _lib.apb_block_attention_hosts.argtypes
_lib.apb_block_attention_range.restype = ctypes.c_int
_lib.apb_block_attention_host_set.argtypes = ([ctypes.POINTER(Config)] + [ctypes.c_int32] * 3
                                              + [_P] * 8 + [ctypes.c_size_t, _P])
_lib.apb_block_attention_host_set.restype = ctypes.c_int
_lib.apb_score_compress_static.argtypes = [ctypes.POINTER(Config)] + [_P] * 9
_lib.apb_score_compress_static.restype = ctypes.c_int
_lib.apb_score_compress_static_max_floats.argtypes = []
_lib.apb_score_compress_static_max_floats.restype = ctypes.c_size_t
_lib.apb_score_compress_static_status.argtypes = [_P, ctypes.c_int]
_lib.apb_score_compress_static_status.restype = ctypes.c_int
_lib.apb_score_compress_static_selftest.argtypes = [ctypes.c_uint32, _P]
_lib.apb_score_compress_static_selftest.restype = ctypes.c_int
_lib.apb_selftest_set_wait_limit.argtypes = [ctypes.c_uint64]
_lib.apb_selftest_set_wait_limit.restype = ctypes.c_int
_lib.apb_selftest_wait_timeout.argtypes = [_P, ctypes.c_size_t, ctypes.c_uint32, _P]
_lib.apb_selftest_wait_timeout.restype = ctypes.c_int
_lib.apb_device_status.argtypes = [_P, _P, ctypes.c_int]
_lib.apb_device_status.restype = ctypes.c_int
_lib.apb_status_string.argtypes = [ctypes.c_int]
_lib.apb_status_string.restype = ctypes.c_char_p
_lib.apb_last_error.argtypes = []
_lib.apb_last_error.restype = ctypes.c_char_p


class APBError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = _lib.apb_status_string(status).decode()
        detail = _lib.apb_last_error().decode()
        super().__init__(f"{where}: {name}: {detail}")


def _check(status: int, where: str) -> None:
    if status != APB_OK:
        raise APBError(status, where)


def status_string(status: int) -> str:
    return _lib.apb_status_string(status).decode()


def declared_symbols() -> list:
    """Entry points declared in include/apb.h."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"\b(apb_[a-z_]+)\s*\(", text)))


def make_config(cfg=None, **kw) -> Config:
    """apb_config from an ``inputs.APBConfig`` (or keyword fields)."""
    f = {}
    if cfg is not None:
        f = dict(n_hosts=cfg.n_hosts, block_len=cfg.block_len, anchor_len=cfg.anchor_len,
                 query_len=cfg.query_len, keep=cfg.keep, n_q_heads=cfg.n_q_heads,
                 n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim, mlp_hidden=cfg.mlp_hidden,
                 softmax_scale=0.0)
    f.update(kw)
    f.setdefault("mlp_hidden", 256)
    f.setdefault("softmax_scale", 0.0)
    return Config(**f)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _want(t: torch.Tensor, name: str, dtype, shape) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _dims(c: Config):
    N = c.n_hosts * c.block_len
    return N, c.n_q_heads, c.n_kv_heads, c.head_dim


def workspace_bytes(c: Config) -> int:
    return int(_lib.apb_workspace_bytes(ctypes.byref(c)))


def new_workspace(c: Config, device="cuda") -> torch.Tensor:
    """Zero-filled device workspace of apb_workspace_bytes(c) bytes."""
    n = workspace_bytes(c)
    if n == 0:
        _check(APB_ERR_INVALID_ARG, "apb_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def score_compress(c: Config, q, k, v, w1, b1, w2, b2, scores=None, idx=None, workspace=None,
                   stream=None, query_aware=False) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """apb_score_compress (or apb_score_compress_query_aware when
    query_aware): returns (idx [H, Hkv, keep] int32, scores or None)."""
    N, hq, hkv, d = _dims(c)
    _want(q, "q", torch.bfloat16, (N, hq, d))
    _want(k, "k", torch.bfloat16, (N, hkv, d))
    _want(v, "v", torch.bfloat16, (N, hkv, d))
    _want(w1, "w1", torch.float32, (hkv, c.mlp_hidden, 3 * d))
    _want(b1, "b1", torch.float32, (hkv, c.mlp_hidden))
    _want(w2, "w2", torch.float32, (hkv, c.mlp_hidden))
    _want(b2, "b2", torch.float32, (hkv,))
    if scores is not None:
        _want(scores, "scores", torch.float32, (hkv, N))
    if idx is None:
        idx = torch.empty((c.n_hosts, hkv, c.keep), dtype=torch.int32, device=q.device)
    _want(idx, "idx", torch.int32, (c.n_hosts, hkv, c.keep))
    if workspace is None:
        workspace = new_workspace(c, q.device)
    fn = _lib.apb_score_compress_query_aware if query_aware else _lib.apb_score_compress
    st = fn(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2),
            _ptr(scores), _ptr(idx) if idx.numel() else None, _ptr(workspace), workspace.numel(),
            _stream(stream))
    _check(st, "apb_score_compress_query_aware" if query_aware else "apb_score_compress")
    return idx, scores


def score_compress_pass(c: Config, q, k, v, w1, b1, w2, b2, pass_k, pass_v, scores=None,
                        idx=None, workspace=None, stream=None) -> torch.Tensor:
    """apb_score_compress_pass: score, top-k and the passing-block gather (the
    gather in the top-k launch); fills pass_k / pass_v [H*keep, Hkv, d] and
    returns idx [H, Hkv, keep] int32."""
    N, hq, hkv, d = _dims(c)
    _want(q, "q", torch.bfloat16, (N, hq, d))
    _want(k, "k", torch.bfloat16, (N, hkv, d))
    _want(v, "v", torch.bfloat16, (N, hkv, d))
    _want(w1, "w1", torch.float32, (hkv, c.mlp_hidden, 3 * d))
    _want(b1, "b1", torch.float32, (hkv, c.mlp_hidden))
    _want(w2, "w2", torch.float32, (hkv, c.mlp_hidden))
    _want(b2, "b2", torch.float32, (hkv,))
    _want(pass_k, "pass_k", torch.bfloat16, (c.n_hosts * c.keep, hkv, d))
    _want(pass_v, "pass_v", torch.bfloat16, (c.n_hosts * c.keep, hkv, d))
    if scores is not None:
        _want(scores, "scores", torch.float32, (hkv, N))
    if idx is None:
        idx = torch.empty((c.n_hosts, hkv, c.keep), dtype=torch.int32, device=q.device)
    _want(idx, "idx", torch.int32, (c.n_hosts, hkv, c.keep))
    if workspace is None:
        workspace = new_workspace(c, q.device)
    has = idx.numel() > 0
    st = _lib.apb_score_compress_pass(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), _ptr(w1),
                                      _ptr(b1), _ptr(w2), _ptr(b2), _ptr(scores),
                                      _ptr(idx) if has else None, _ptr(pass_k) if has else None,
                                      _ptr(pass_v) if has else None, _ptr(workspace),
                                      workspace.numel(), _stream(stream))
    _check(st, "apb_score_compress_pass")
    return idx


def score_compress_static(c: Config, q, k, v, w1, b1, w2, b2, idx=None, stream=None):
    """apb_score_compress_static: the allocation-free variant (scores kept in
    the library's fixed device array); returns idx [H, Hkv, keep] int32."""
    N, hq, hkv, d = _dims(c)
    _want(q, "q", torch.bfloat16, (N, hq, d))
    _want(k, "k", torch.bfloat16, (N, hkv, d))
    _want(v, "v", torch.bfloat16, (N, hkv, d))
    _want(w1, "w1", torch.float32, (hkv, c.mlp_hidden, 3 * d))
    _want(b1, "b1", torch.float32, (hkv, c.mlp_hidden))
    _want(w2, "w2", torch.float32, (hkv, c.mlp_hidden))
    _want(b2, "b2", torch.float32, (hkv,))
    if idx is None:
        idx = torch.empty((c.n_hosts, hkv, c.keep), dtype=torch.int32, device=q.device)
    _want(idx, "idx", torch.int32, (c.n_hosts, hkv, c.keep))
    st = _lib.apb_score_compress_static(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), _ptr(w1),
                                        _ptr(b1), _ptr(w2), _ptr(b2),
                                        _ptr(idx) if idx.numel() else None, _stream(stream))
    _check(st, "apb_score_compress_static")
    return idx


def score_compress_static_status(stream=None, clear=False) -> int:
    """apb_score_compress_static_status: synchronises the stream and returns
    APB_ERR_TIMEOUT if a wait inside apb_score_compress_static ran out."""
    return int(_lib.apb_score_compress_static_status(_stream(stream), 1 if clear else 0))


def score_compress_static_selftest(limit_us: int, stream=None):
    """apb_score_compress_static_selftest: the bounded-wait self-test on the
    static entry point's own status block."""
    st = _lib.apb_score_compress_static_selftest(limit_us, _stream(stream))
    _check(st, "apb_score_compress_static_selftest")


def build_passing(c: Config, k, v, idx, pass_k=None, pass_v=None, stream=None):
    """apb_build_passing: returns (pass_k, pass_v) [H*keep, Hkv, d] bf16."""
    N, hq, hkv, d = _dims(c)
    _want(k, "k", torch.bfloat16, (N, hkv, d))
    _want(v, "v", torch.bfloat16, (N, hkv, d))
    _want(idx, "idx", torch.int32, (c.n_hosts, hkv, c.keep))
    shape = (c.n_hosts * c.keep, hkv, d)
    if pass_k is None:
        pass_k = torch.empty(shape, dtype=torch.bfloat16, device=k.device)
    if pass_v is None:
        pass_v = torch.empty(shape, dtype=torch.bfloat16, device=k.device)
    _want(pass_k, "pass_k", torch.bfloat16, shape)
    _want(pass_v, "pass_v", torch.bfloat16, shape)
    if c.keep == 0:
        return pass_k, pass_v
    st = _lib.apb_build_passing(ctypes.byref(c), _ptr(k), _ptr(v), _ptr(idx), _ptr(pass_k),
                                _ptr(pass_v), _stream(stream))
    _check(st, "apb_build_passing")
    return pass_k, pass_v


def block_attention(c: Config, q, k, v, pass_k, pass_v, out=None, lse=None, want_lse=False,
                    workspace=None, stream=None):
    """apb_block_attention: returns (out [N, Hq, d] bf16, lse [Hq, N] fp32 or None)."""
    N, hq, hkv, d = _dims(c)
    _want(q, "q", torch.bfloat16, (N, hq, d))
    _want(k, "k", torch.bfloat16, (N, hkv, d))
    _want(v, "v", torch.bfloat16, (N, hkv, d))
    use_pass = c.keep > 0 and c.n_hosts > 1
    if use_pass:
        shape = (c.n_hosts * c.keep, hkv, d)
        _want(pass_k, "pass_k", torch.bfloat16, shape)
        _want(pass_v, "pass_v", torch.bfloat16, shape)
    if out is None:
        out = torch.empty((N, hq, d), dtype=torch.bfloat16, device=q.device)
    _want(out, "out", torch.bfloat16, (N, hq, d))
    if lse is None and want_lse:
        lse = torch.empty((hq, N), dtype=torch.float32, device=q.device)
    if lse is not None:
        _want(lse, "lse", torch.float32, (hq, N))
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=q.device)
    st = _lib.apb_block_attention(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(pass_k) if use_pass else None,
                                  _ptr(pass_v) if use_pass else None, _ptr(out), _ptr(lse),
                                  _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "apb_block_attention")
    return out, lse


def block_attention_range(c: Config, host_begin: int, host_end: int, q, k, v, pass_k, pass_v,
                          out, lse=None, workspace=None, stream=None):
    """apb_block_attention_range: attention of hosts [host_begin, host_end)
    on the whole-sequence buffers; writes only those hosts' rows of out (and
    lse).  Returns (out, lse)."""
    N, hq, hkv, d = _dims(c)
    _want(q, "q", torch.bfloat16, (N, hq, d))
    _want(k, "k", torch.bfloat16, (N, hkv, d))
    _want(v, "v", torch.bfloat16, (N, hkv, d))
    _want(out, "out", torch.bfloat16, (N, hq, d))
    use_pass = c.keep > 0 and host_end > 1
    if use_pass:
        shape = (c.n_hosts * c.keep, hkv, d)
        _want(pass_k, "pass_k", torch.bfloat16, shape)
        _want(pass_v, "pass_v", torch.bfloat16, shape)
    if lse is not None:
        _want(lse, "lse", torch.float32, (hq, N))
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=q.device)
    st = _lib.apb_block_attention_range(ctypes.byref(c), host_begin, host_end, _ptr(q), _ptr(k),
                                        _ptr(v), _ptr(pass_k) if use_pass else None,
                                        _ptr(pass_v) if use_pass else None, _ptr(out), _ptr(lse),
                                        _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "apb_block_attention_range")
    return out, lse


def block_attention_hosts(c: Config, host_begin: int, host_end: int, q, kv_k, kv_v, pass_k,
                          pass_v, out=None, lse=None, want_lse=False, workspace=None,
                          stream=None):
    """apb_block_attention_hosts: attention of hosts [host_begin, host_end)
    on rank-local buffers (q/out: those hosts' rows; kv_k/kv_v: the anchor's
    rows, then those hosts' rows).  Returns (out, lse or None)."""
    _, hq, hkv, d = _dims(c)
    rows = (host_end - host_begin) * c.block_len
    _want(q, "q", torch.bfloat16, (rows, hq, d))
    _want(kv_k, "kv_k", torch.bfloat16, (c.anchor_len + rows, hkv, d))
    _want(kv_v, "kv_v", torch.bfloat16, (c.anchor_len + rows, hkv, d))
    use_pass = c.keep > 0 and host_end > 1
    if use_pass:
        shape = (c.n_hosts * c.keep, hkv, d)
        _want(pass_k, "pass_k", torch.bfloat16, shape)
        _want(pass_v, "pass_v", torch.bfloat16, shape)
    if out is None:
        out = torch.empty((rows, hq, d), dtype=torch.bfloat16, device=q.device)
    _want(out, "out", torch.bfloat16, (rows, hq, d))
    if lse is None and want_lse:
        lse = torch.empty((hq, rows), dtype=torch.float32, device=q.device)
    if lse is not None:
        _want(lse, "lse", torch.float32, (hq, rows))
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=q.device)
    st = _lib.apb_block_attention_hosts(ctypes.byref(c), host_begin, host_end, _ptr(q), _ptr(kv_k),
                                        _ptr(kv_v), _ptr(pass_k) if use_pass else None,
                                        _ptr(pass_v) if use_pass else None, _ptr(out), _ptr(lse),
                                        _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "apb_block_attention_hosts")
    return out, lse


def block_attention_host_set(c: Config, host_first: int, host_count: int, host_stride: int, q,
                             kv_k, kv_v, pass_k, pass_v, out=None, lse=None, want_lse=False,
                             workspace=None, stream=None):
    """apb_block_attention_host_set: attention of the hosts host_first +
    i*host_stride, i < host_count, on rank-local buffers (q/out: those hosts'
    rows in order; kv_k/kv_v: the anchor's rows, then those hosts' rows).
    Returns (out, lse or None)."""
    _, hq, hkv, d = _dims(c)
    rows = host_count * c.block_len
    _want(q, "q", torch.bfloat16, (rows, hq, d))
    _want(kv_k, "kv_k", torch.bfloat16, (c.anchor_len + rows, hkv, d))
    _want(kv_v, "kv_v", torch.bfloat16, (c.anchor_len + rows, hkv, d))
    use_pass = c.keep > 0 and host_first + (host_count - 1) * host_stride >= 1
    if use_pass:
        shape = (c.n_hosts * c.keep, hkv, d)
        _want(pass_k, "pass_k", torch.bfloat16, shape)
        _want(pass_v, "pass_v", torch.bfloat16, shape)
    if out is None:
        out = torch.empty((rows, hq, d), dtype=torch.bfloat16, device=q.device)
    _want(out, "out", torch.bfloat16, (rows, hq, d))
    if lse is None and want_lse:
        lse = torch.empty((hq, rows), dtype=torch.float32, device=q.device)
    if lse is not None:
        _want(lse, "lse", torch.float32, (hq, rows))
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=q.device)
    st = _lib.apb_block_attention_host_set(ctypes.byref(c), host_first, host_count, host_stride,
                                           _ptr(q), _ptr(kv_k), _ptr(kv_v),
                                           _ptr(pass_k) if use_pass else None,
                                           _ptr(pass_v) if use_pass else None, _ptr(out),
                                           _ptr(lse), _ptr(workspace), workspace.numel(),
                                           _stream(stream))
    _check(st, "apb_block_attention_host_set")
    return out, lse


def prefill_workspace_bytes(c: Config) -> int:
    return int(_lib.apb_prefill_workspace_bytes(ctypes.byref(c)))


def prefill(c: Config, q, k, v, w1, b1, w2, b2, out=None, lse=None, want_lse=False,
            workspace=None, stream=None):
    """apb_prefill: the whole path in one call.  Returns (out, lse or None)."""
    N, hq, hkv, d = _dims(c)
    _want(q, "q", torch.bfloat16, (N, hq, d))
    _want(k, "k", torch.bfloat16, (N, hkv, d))
    _want(v, "v", torch.bfloat16, (N, hkv, d))
    _want(w1, "w1", torch.float32, (hkv, c.mlp_hidden, 3 * d))
    _want(b1, "b1", torch.float32, (hkv, c.mlp_hidden))
    _want(w2, "w2", torch.float32, (hkv, c.mlp_hidden))
    _want(b2, "b2", torch.float32, (hkv,))
    if out is None:
        out = torch.empty((N, hq, d), dtype=torch.bfloat16, device=q.device)
    _want(out, "out", torch.bfloat16, (N, hq, d))
    if lse is None and want_lse:
        lse = torch.empty((hq, N), dtype=torch.float32, device=q.device)
    if lse is not None:
        _want(lse, "lse", torch.float32, (hq, N))
    if workspace is None:
        workspace = torch.zeros(prefill_workspace_bytes(c), dtype=torch.uint8, device=q.device)
    st = _lib.apb_prefill(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), _ptr(w1), _ptr(b1),
                          _ptr(w2), _ptr(b2), _ptr(out), _ptr(lse), _ptr(workspace),
                          workspace.numel(), _stream(stream))
    _check(st, "apb_prefill")
    return out, lse


def device_status(workspace, stream=None, clear=False) -> int:
    """apb_device_status: synchronises the stream, returns the status code."""
    return int(_lib.apb_device_status(_ptr(workspace), _stream(stream), 1 if clear else 0))


def selftest_wait_timeout(workspace, limit_us: int, stream=None):
    """apb_selftest_wait_timeout: two CTAs wait on barriers that nothing
    completes; returns the launch status.  Read the outcome with
    device_status(); the two waits' elapsed nanoseconds are bytes 64..79 of
    the workspace."""
    st = _lib.apb_selftest_wait_timeout(_ptr(workspace), workspace.numel(), limit_us,
                                        _stream(stream))
    _check(st, "apb_selftest_wait_timeout")


def selftest_set_wait_limit(limit_ns: int):
    """apb_selftest_set_wait_limit: time limit of the kernels' bounded waits
    for later launches (0 restores the default 1 s)."""
    _check(_lib.apb_selftest_set_wait_limit(limit_ns), "apb_selftest_set_wait_limit")


class Prefill:
    """One APB prefill over preallocated device buffers: score + compress
    with the passing block built in the top-k launch, then block attention.  Buffers are allocated once (by
    torch) and reused by every call."""

    def __init__(self, c: Config, device="cuda"):
        N, hq, hkv, d = _dims(c)
        self.c = c
        self.workspace = new_workspace(c, device)
        self.idx = torch.empty((c.n_hosts, hkv, c.keep), dtype=torch.int32, device=device)
        shape = (c.n_hosts * c.keep, hkv, d)
        self.pass_k = torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.pass_v = torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.out = torch.empty((N, hq, d), dtype=torch.bfloat16, device=device)

    def __call__(self, q, k, v, w1, b1, w2, b2, stream=None):
        score_compress_pass(self.c, q, k, v, w1, b1, w2, b2, self.pass_k, self.pass_v,
                            idx=self.idx, workspace=self.workspace, stream=stream)
        block_attention(self.c, q, k, v, self.pass_k, self.pass_v, out=self.out,
                        workspace=self.workspace, stream=stream)
        return self.out


class PrefillPipeline:
    """Prefills of successive sequences from pinned host memory with the
    transfers of one step overlapped with the compute of another.

    Each of `depth` slots owns device copies of the inputs, an apb_prefill
    workspace and an output buffer; the compute is one apb_prefill call.  submit() queues, on three
    streams ordered by events, the host->device copy of the step's inputs,
    the three calls of the path, and the device->host copy of the output into
    the caller's pinned buffer.  A slot's inputs are overwritten only after its
    previous compute has finished, and its output only after the previous copy
    back has finished.  synchronize() waits for everything queued."""

    def __init__(self, c: Config, device="cuda", depth: int = 2):
        N, hq, hkv, d = _dims(c)
        dev = torch.device(device)
        self.c = c
        self.depth = depth
        self.h2d = torch.cuda.Stream(dev)
        self.comp = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        self.slots = []
        for _ in range(depth):
            x = {"q": torch.empty((N, hq, d), dtype=torch.bfloat16, device=dev),
                 "k": torch.empty((N, hkv, d), dtype=torch.bfloat16, device=dev),
                 "v": torch.empty((N, hkv, d), dtype=torch.bfloat16, device=dev),
                 "w1": torch.empty((hkv, c.mlp_hidden, 3 * d), dtype=torch.float32, device=dev),
                 "b1": torch.empty((hkv, c.mlp_hidden), dtype=torch.float32, device=dev),
                 "w2": torch.empty((hkv, c.mlp_hidden), dtype=torch.float32, device=dev),
                 "b2": torch.empty((hkv,), dtype=torch.float32, device=dev)}
            ev = {k: torch.cuda.Event() for k in ("in", "comp", "out")}
            self.slots.append({"x": x, "ev": ev, "used": False,
                               "ws": torch.zeros(prefill_workspace_bytes(c), dtype=torch.uint8,
                                                 device=dev),
                               "out": torch.empty((N, hq, d), dtype=torch.bfloat16, device=dev)})
        self.i = 0

    def submit(self, host: dict, host_out: torch.Tensor) -> None:
        """host: pinned CPU tensors q, k, v, w1, b1, w2, b2; host_out: pinned
        CPU bf16 [N, Hq, d] receiving this step's output."""
        slot = self.slots[self.i % self.depth]
        self.i += 1
        ev = slot["ev"]
        with torch.cuda.stream(self.h2d):
            if slot["used"]:
                self.h2d.wait_event(ev["comp"])          # previous compute done reading
            for k, t in slot["x"].items():
                t.copy_(host[k], non_blocking=True)
            ev["in"].record(self.h2d)
        with torch.cuda.stream(self.comp):
            self.comp.wait_event(ev["in"])
            if slot["used"]:
                self.comp.wait_event(ev["out"])          # previous output copied back
            x = slot["x"]
            prefill(self.c, x["q"], x["k"], x["v"], x["w1"], x["b1"], x["w2"], x["b2"],
                    out=slot["out"], workspace=slot["ws"], stream=self.comp)
            ev["comp"].record(self.comp)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(ev["comp"])
            host_out.copy_(slot["out"], non_blocking=True)
            ev["out"].record(self.d2h)
        slot["used"] = True

    def synchronize(self) -> None:
        for st in (self.h2d, self.comp, self.d2h):
            st.synchronize()


class StreamedPrefill:
    """Prefills of successive sequences from pinned host memory, streamed host
    by host: host h's rows are copied in, compressed and attended while the
    rows of later hosts are still on their way, and its output rows go back as
    soon as they are done.  So a step's copies overlap its own compute, not
    only another step's, and the first copy-in and last copy-out of a run
    cost one host's rows instead of a whole sequence.

    Per step (streams ordered by events): the H2D stream copies the weights,
    then host 0, 1, ... (q, k, v rows); one compute stream compresses host h
    (apb_score_compress_pass on host h's rows with a one-host config,
    writing rows [h*keep, (h+1)*keep) of the passing buffers) once its rows are in; two attention streams take hosts in turn
    (apb_block_attention_range for host h once its rows and the compressed
    blocks of hosts 0..h-1 are in place), so one host's launch fills the
    tail of the other's; the D2H stream copies host h's output rows out.
    The last host's compression is skipped (no host follows it).  `depth`
    slots own the device buffers; a slot is reused only after all its work,
    including the copy-out, has finished.  synchronize() waits for
    everything queued."""

    def __init__(self, c: Config, device="cuda", depth: int = 2):
        N, hq, hkv, d = _dims(c)
        dev = torch.device(device)
        self.c = c
        self.depth = depth
        self.H, self.n = c.n_hosts, c.block_len
        self.c1 = make_config(None, n_hosts=1, block_len=c.block_len, anchor_len=c.anchor_len,
                              query_len=c.query_len, keep=c.keep, n_q_heads=c.n_q_heads,
                              n_kv_heads=c.n_kv_heads, head_dim=c.head_dim,
                              mlp_hidden=c.mlp_hidden, softmax_scale=c.softmax_scale)
        self.h2d = torch.cuda.Stream(dev)
        self.comp = torch.cuda.Stream(dev)
        self.att = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
        self.d2h = torch.cuda.Stream(dev)
        self.slots = []
        for _ in range(depth):
            x = {"q": torch.empty((N, hq, d), dtype=torch.bfloat16, device=dev),
                 "k": torch.empty((N, hkv, d), dtype=torch.bfloat16, device=dev),
                 "v": torch.empty((N, hkv, d), dtype=torch.bfloat16, device=dev),
                 "w1": torch.empty((hkv, c.mlp_hidden, 3 * d), dtype=torch.float32, device=dev),
                 "b1": torch.empty((hkv, c.mlp_hidden), dtype=torch.float32, device=dev),
                 "w2": torch.empty((hkv, c.mlp_hidden), dtype=torch.float32, device=dev),
                 "b2": torch.empty((hkv,), dtype=torch.float32, device=dev)}
            shape = (max(self.H, 1) * c.keep, hkv, d)
            self.slots.append({
                "x": x, "used": False,
                "out": torch.empty((N, hq, d), dtype=torch.bfloat16, device=dev),
                "idx": torch.empty((self.H, 1, hkv, c.keep), dtype=torch.int32, device=dev),
                "pass_k": torch.empty(shape, dtype=torch.bfloat16, device=dev),
                "pass_v": torch.empty(shape, dtype=torch.bfloat16, device=dev),
                "ws_comp": new_workspace(self.c1, dev),
                "ws_att": [torch.zeros(256, dtype=torch.uint8, device=dev) for _ in range(2)],
                "ev_in": [torch.cuda.Event() for _ in range(self.H)],
                "ev_pass": [torch.cuda.Event() for _ in range(self.H)],
                "ev_att": [torch.cuda.Event() for _ in range(self.H)],
                "ev_done": [torch.cuda.Event() for _ in range(4)],   # comp, att0, att1, d2h
            })
        self.i = 0

    def workspaces(self):
        """Every workspace (for apb_device_status)."""
        return [w for sl in self.slots for w in [sl["ws_comp"]] + sl["ws_att"]]

    def submit(self, host: dict, host_out: torch.Tensor) -> None:
        """host: pinned CPU tensors q, k, v, w1, b1, w2, b2; host_out: pinned
        CPU bf16 [N, Hq, d] receiving this step's output."""
        sl = self.slots[self.i % self.depth]
        self.i += 1
        H, n, keep = self.H, self.n, self.c.keep
        x = sl["x"]
        compress = keep > 0 and H > 1
        with torch.cuda.stream(self.h2d):
            if sl["used"]:
                for e in sl["ev_done"]:              # the slot's previous step is over
                    self.h2d.wait_event(e)
            for name in ("w1", "b1", "w2", "b2"):
                x[name].copy_(host[name], non_blocking=True)
            for h in range(H):
                rows = slice(h * n, (h + 1) * n)
                for name in ("q", "k", "v"):
                    x[name][rows].copy_(host[name][rows], non_blocking=True)
                sl["ev_in"][h].record(self.h2d)
        with torch.cuda.stream(self.comp):
            if compress:
                for h in range(H - 1):
                    rows = slice(h * n, (h + 1) * n)
                    self.comp.wait_event(sl["ev_in"][h])
                    score_compress_pass(self.c1, x["q"][rows], x["k"][rows], x["v"][rows],
                                        x["w1"], x["b1"], x["w2"], x["b2"],
                                        sl["pass_k"][h * keep:(h + 1) * keep],
                                        sl["pass_v"][h * keep:(h + 1) * keep], idx=sl["idx"][h],
                                        workspace=sl["ws_comp"], stream=self.comp)
                    sl["ev_pass"][h].record(self.comp)
            sl["ev_done"][0].record(self.comp)
        for h in range(H):
            s = self.att[h % 2]
            with torch.cuda.stream(s):
                s.wait_event(sl["ev_in"][h])
                if compress and h >= 1:
                    s.wait_event(sl["ev_pass"][h - 1])
                block_attention_range(self.c, h, h + 1, x["q"], x["k"], x["v"], sl["pass_k"],
                                      sl["pass_v"], sl["out"], workspace=sl["ws_att"][h % 2],
                                      stream=s)
                sl["ev_att"][h].record(s)
        for j, s in enumerate(self.att):
            sl["ev_done"][1 + j].record(s)
        with torch.cuda.stream(self.d2h):
            for h in range(H):
                rows = slice(h * n, (h + 1) * n)
                self.d2h.wait_event(sl["ev_att"][h])
                host_out[rows].copy_(sl["out"][rows], non_blocking=True)
            sl["ev_done"][3].record(self.d2h)
        sl["used"] = True

    def synchronize(self) -> None:
        for st in [self.h2d, self.comp, self.d2h] + self.att:
            st.synchronize()

"""The C-ABI library loads, exports every entry point include/apb.h declares,
and rejects bad arguments on the host before launching anything (no GPU is
needed: every case here returns before the first CUDA call)."""
import ctypes
import subprocess

import pytest

from long_context_sparse_apb_b200 import _lib as apb
from long_context_sparse_apb_b200 import inputs


def test_every_declared_symbol_is_exported():
    names = apb.declared_symbols()
    assert set(names) >= {"apb_score_compress", "apb_build_passing", "apb_block_attention",
                          "apb_workspace_bytes", "apb_status_string", "apb_device_status",
                          "apb_last_error"}
    out = subprocess.run(["nm", "-D", "--defined-only", apb.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, n
        assert hasattr(apb._lib, n)


def test_status_strings():
    assert apb.status_string(0) == "APB_OK"
    assert apb.status_string(1) == "APB_ERR_INVALID_ARG"
    assert apb.status_string(4) == "APB_ERR_TIMEOUT"
    assert apb.status_string(99) == "APB_ERR_UNKNOWN"


def test_workspace_bytes():
    c = apb.make_config(inputs.LLAMA8B_128K)
    assert apb.workspace_bytes(c) == 256 + 8 * 256 * 384 * 4 + 8 * 256 * 4 + 8 * 131072 * 4
    bad = apb.make_config(inputs.TINY, keep=10_000)
    assert apb.workspace_bytes(bad) == 0
    assert apb._lib.apb_workspace_bytes(None) == 0


FAKE = ctypes.c_void_p(1 << 20)          # aligned, never dereferenced
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)


def _attn(c, q=FAKE, out=FAKE, ws=FAKE, wsb=256):
    return apb._lib.apb_block_attention(ctypes.byref(c), q, FAKE, FAKE, FAKE, FAKE, out, None,
                                        ws, wsb, None)


@pytest.mark.parametrize("field,value,code", [
    ("n_hosts", 0, apb.APB_ERR_INVALID_ARG),
    ("block_len", 0, apb.APB_ERR_INVALID_ARG),
    ("anchor_len", 600, apb.APB_ERR_INVALID_ARG),     # A > n
    ("query_len", 200, apb.APB_ERR_INVALID_ARG),      # q_len > A
    ("keep", 513, apb.APB_ERR_INVALID_ARG),           # keep > n
    ("keep", -1, apb.APB_ERR_INVALID_ARG),
    ("n_q_heads", 5, apb.APB_ERR_INVALID_ARG),        # not a multiple of Hkv
    ("head_dim", 96, apb.APB_ERR_UNSUPPORTED),
    ("mlp_hidden", 128, apb.APB_ERR_UNSUPPORTED),
])
def test_invalid_config_rejected(field, value, code):
    c = apb.make_config(inputs.TINY, **{field: value})
    assert _attn(c) == code
    assert apb._lib.apb_build_passing(ctypes.byref(c), FAKE, FAKE, FAKE, FAKE, FAKE, None) == code
    st = apb._lib.apb_score_compress(ctypes.byref(c), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                     None, FAKE, FAKE, 1 << 30, None)
    assert st == code
    assert apb._lib.apb_last_error()


def test_null_and_misaligned_pointers_rejected():
    c = apb.make_config(inputs.TINY)
    assert apb._lib.apb_block_attention(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 256,
                                        None) == apb.APB_ERR_INVALID_ARG
    assert _attn(c, q=None) == apb.APB_ERR_INVALID_ARG
    assert _attn(c, out=MISALIGNED) == apb.APB_ERR_INVALID_ARG
    assert _attn(c, ws=None) == apb.APB_ERR_INVALID_ARG
    assert _attn(c, wsb=64) == apb.APB_ERR_INVALID_ARG
    # passing block required when keep > 0 and H > 1
    st = apb._lib.apb_block_attention(ctypes.byref(c), FAKE, FAKE, FAKE, None, None, FAKE, None,
                                      FAKE, 256, None)
    assert st == apb.APB_ERR_INVALID_ARG
    # score_compress: workspace too small to hold the scores when scores is NULL
    st = apb._lib.apb_score_compress(ctypes.byref(c), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                     None, FAKE, FAKE, 256, None)
    assert st == apb.APB_ERR_INVALID_ARG
    st = apb._lib.apb_build_passing(ctypes.byref(c), FAKE, FAKE, None, FAKE, FAKE, None)
    assert st == apb.APB_ERR_INVALID_ARG
    assert apb._lib.apb_device_status(None, None, 0) == apb.APB_ERR_INVALID_ARG


def test_keep_zero_build_passing_is_a_no_op():
    c = apb.make_config(inputs.TINY, keep=0)
    assert apb._lib.apb_build_passing(ctypes.byref(c), None, None, None, None, None, None) == 0


def test_selftest_argument_checks():
    assert apb._lib.apb_selftest_wait_timeout(None, 256, 1000, None) == apb.APB_ERR_INVALID_ARG
    assert apb._lib.apb_selftest_wait_timeout(FAKE, 64, 1000, None) == apb.APB_ERR_INVALID_ARG
    assert apb._lib.apb_selftest_wait_timeout(FAKE, 256, 0, None) == apb.APB_ERR_INVALID_ARG
    assert apb._lib.apb_selftest_wait_timeout(FAKE, 256, 2_000_000, None) == apb.APB_ERR_INVALID_ARG


def test_prefill_workspace_and_checks():
    c = apb.make_config(inputs.LLAMA8B_128K)
    H, n, hkv, keep, d = 8, 16384, 8, 2048, 128
    r = lambda x: (x + 255) // 256 * 256
    expect = (256 + r(hkv * 256 * 384 * 4) + r(hkv * 256 * 4) + r((H - 1) * n * hkv * 4)
              + r((H - 1) * hkv * keep * 4) + 2 * r(H * keep * hkv * d * 2))
    assert apb.prefill_workspace_bytes(c) == expect
    st = apb._lib.apb_prefill(ctypes.byref(c), *([FAKE] * 7), None, None, FAKE, 1 << 40, None)
    assert st == apb.APB_ERR_INVALID_ARG                  # out is NULL
    st = apb._lib.apb_prefill(ctypes.byref(c), *([FAKE] * 8), None, FAKE, 256, None)
    assert st == apb.APB_ERR_INVALID_ARG                  # workspace too small


def test_host_range_and_query_aware_checks():
    c = apb.make_config(inputs.TINY)
    args = [FAKE] * 6 + [None, FAKE, 256, None]
    for hb, he in ((0, 0), (2, 1), (-1, 2), (0, 5)):
        assert apb._lib.apb_block_attention_hosts(ctypes.byref(c), hb, he, *args) == \
            apb.APB_ERR_INVALID_ARG
    st = apb._lib.apb_block_attention_hosts(ctypes.byref(c), 1, 3, None, *([FAKE] * 5), None,
                                            FAKE, 256, None)
    assert st == apb.APB_ERR_INVALID_ARG                  # q is NULL
    for hb, he in ((0, 0), (2, 1), (-1, 2), (0, 5)):
        assert apb._lib.apb_block_attention_range(ctypes.byref(c), hb, he, *args) == \
            apb.APB_ERR_INVALID_ARG
    # strided host sets (TINY has 4 hosts): the last host must exist, count and
    # stride must be positive
    for first, count, stride in ((0, 0, 1), (0, 2, 0), (-1, 2, 1), (1, 2, 3), (0, 5, 1),
                                 (3, 2, 1)):
        assert apb._lib.apb_block_attention_host_set(ctypes.byref(c), first, count, stride,
                                                     *args) == apb.APB_ERR_INVALID_ARG
    # the query-aware variant needs room for its bias next to the weight split
    st = apb._lib.apb_score_compress_query_aware(ctypes.byref(c), *([FAKE] * 8), FAKE, FAKE,
                                                 256 + 2 * 256 * 192 * 4, None)
    assert st == apb.APB_ERR_INVALID_ARG
    bad = apb.make_config(inputs.TINY, head_dim=80)
    st = apb._lib.apb_score_compress_query_aware(ctypes.byref(bad), *([FAKE] * 8), FAKE, FAKE,
                                                 1 << 30, None)
    assert st == apb.APB_ERR_UNSUPPORTED


def test_score_compress_pass_checks():
    # the fused call takes the score call's checks plus its own on the
    # passing buffers, all before any launch
    c = apb.make_config(inputs.TINY)
    ws = apb.workspace_bytes(c)
    args = [FAKE] * 8   # q, k, v, w1, b1, w2, b2, scores
    st = apb._lib.apb_score_compress_pass(ctypes.byref(c), *args, FAKE, None, FAKE, FAKE, ws, None)
    assert st == apb.APB_ERR_INVALID_ARG                       # pass_k NULL
    st = apb._lib.apb_score_compress_pass(ctypes.byref(c), *args, FAKE, FAKE, MISALIGNED, FAKE,
                                          ws, None)
    assert st == apb.APB_ERR_INVALID_ARG                       # pass_v misaligned
    st = apb._lib.apb_score_compress_pass(ctypes.byref(c), *args, None, FAKE, FAKE, FAKE, ws, None)
    assert st == apb.APB_ERR_INVALID_ARG                       # idx NULL with keep > 0
    bad = apb.make_config(inputs.TINY, head_dim=96)
    st = apb._lib.apb_score_compress_pass(ctypes.byref(bad), *args, FAKE, FAKE, FAKE, FAKE, ws,
                                          None)
    assert st == apb.APB_ERR_UNSUPPORTED
    st = apb._lib.apb_score_compress_pass(ctypes.byref(c), *args, FAKE, FAKE, FAKE, FAKE, 64, None)
    assert st == apb.APB_ERR_INVALID_ARG                       # workspace too small

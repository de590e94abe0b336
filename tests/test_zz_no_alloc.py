"""The allocation-free score + top-k entry point (apb_score_compress_static).

Some callers cannot give this library device memory beyond the tensors
themselves (a framework whose allocator owns all device memory and exposes
only inputs and outputs, or a service that must not allocate after start-up).
For them apb_score_compress_static keeps the scores in a fixed array inside
the library.  It must select exactly what apb_score_compress selects; the
check runs twice in a row because the array keeps the previous call's data.

This file is collected last on purpose, so a run that stops at its first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

from long_context_sparse_apb_b200 import inputs


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_point():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_apb_b200 import _lib as apb

    cfgs = [inputs.LLAMA8B_32K, inputs.TINY.replace(n_hosts=3, block_len=700, keep=90,
                                                     anchor_len=175, seed=11)]
    for cfg in cfgs:
        x = inputs.generate(cfg)
        xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
        c = apb.make_config(cfg)
        w = (xd["w1"], xd["b1"], xd["w2"], xd["b2"])
        ref, _ = apb.score_compress(c, xd["q"], xd["k"], xd["v"], *w)
        for _ in range(2):
            idx = torch.full_like(ref, -1)
            got = apb.score_compress_static(c, xd["q"], xd["k"], xd["v"], *w, idx=idx)
            torch.cuda.synchronize()
            assert torch.equal(got, ref), cfg.name


@pytest.mark.gpu
def test_static_status_reports_a_wait_that_ran_out():
    """A bounded wait that runs out in the static block is reported by
    apb_score_compress_static_status, and a later call still works."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_apb_b200 import _lib as apb

    assert apb.score_compress_static_status(clear=True) == apb.APB_OK
    apb.score_compress_static_selftest(limit_us=20_000)
    assert apb.score_compress_static_status() == apb.APB_ERR_TIMEOUT
    assert "ran out" in apb._lib.apb_last_error().decode()
    assert apb.score_compress_static_status(clear=True) == apb.APB_ERR_TIMEOUT
    assert apb.score_compress_static_status() == apb.APB_OK

    cfg = inputs.TINY
    x = inputs.generate(cfg)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    c = apb.make_config(cfg)
    w = (xd["w1"], xd["b1"], xd["w2"], xd["b2"])
    ref, _ = apb.score_compress(c, xd["q"], xd["k"], xd["v"], *w)
    got = apb.score_compress_static(c, xd["q"], xd["k"], xd["v"], *w)
    assert apb.score_compress_static_status() == apb.APB_OK
    assert torch.equal(got, ref)


def test_static_entry_point_rejects_oversize_and_bad_config():
    from long_context_sparse_apb_b200 import _lib as apb

    last = lambda: apb._lib.apb_last_error().decode()
    assert apb._lib.apb_score_compress_static_max_floats() == 4 << 20
    fake = ctypes.c_void_p(1 << 20)
    big = apb.make_config(inputs.LLAMA8B_1M_512K, n_hosts=17)     # 8 * 557056 floats > 4 Mi
    st = apb._lib.apb_score_compress_static(ctypes.byref(big), *([fake] * 8), None)
    assert st == apb.APB_ERR_UNSUPPORTED
    assert "n_kv_heads*N = 4456448 scores > 4194304" in last()
    # 40 kv heads * 256 * 384 * 4 B = 15.7 MB of split weights > 8 MiB (scores fit)
    wide = apb.make_config(inputs.TINY, n_q_heads=40, n_kv_heads=40, head_dim=128)
    st = apb._lib.apb_score_compress_static(ctypes.byref(wide), *([fake] * 8), None)
    assert st == apb.APB_ERR_UNSUPPORTED
    assert "W1 split 15728640 B > 8388608 B" in last()
    bad = apb.make_config(inputs.TINY, keep=10_000)
    st = apb._lib.apb_score_compress_static(ctypes.byref(bad), *([fake] * 8), None)
    assert st == apb.APB_ERR_INVALID_ARG
    assert "keep(10000)" in last()
    ok = apb.make_config(inputs.TINY)
    st = apb._lib.apb_score_compress_static(ctypes.byref(ok), fake, None, *([fake] * 6), None)
    assert st == apb.APB_ERR_INVALID_ARG
    assert "apb_score_compress_static: NULL input" in last()
    st = apb._lib.apb_score_compress_static_selftest(0, None)
    assert st == apb.APB_ERR_INVALID_ARG
    assert "limit_us=0" in last()

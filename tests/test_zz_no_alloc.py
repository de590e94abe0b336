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


def test_static_entry_point_rejects_oversize_and_bad_config():
    from long_context_sparse_apb_b200 import _lib as apb

    assert apb._lib.apb_score_compress_static_max_floats() == 4 << 20
    fake = ctypes.c_void_p(1 << 20)
    big = apb.make_config(inputs.LLAMA8B_1M_512K, n_hosts=17)     # 8 * 557056 floats > 4 Mi
    st = apb._lib.apb_score_compress_static(ctypes.byref(big), *([fake] * 8), None)
    assert st == apb.APB_ERR_UNSUPPORTED
    bad = apb.make_config(inputs.TINY, keep=10_000)
    st = apb._lib.apb_score_compress_static(ctypes.byref(bad), *([fake] * 8), None)
    assert st == apb.APB_ERR_INVALID_ARG

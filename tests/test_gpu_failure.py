"""Failure detection on the GPU without a fault: a bounded wait that runs out.

apb_selftest_wait_timeout launches two CTAs waiting on barriers that nothing
completes, through the same bounded-wait primitive and status block as the
score and attention kernels.  The short wait must run out, record
APB_ERR_TIMEOUT and stop the other CTA through the launch-wide abort flag long
before its own limit; the context must stay usable afterwards.
"""
import numpy as np
import pytest
import torch

from long_context_sparse_apb_b200 import inputs

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_apb_b200 import _lib as apb

    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    apb.selftest_wait_timeout(ws, limit_us=20_000)
    assert apb.device_status(ws) == apb.APB_ERR_TIMEOUT
    elapsed = ws[64:80].cpu().numpy().view(np.uint64)
    assert 20e6 <= elapsed[0] < 1e9            # ran to its 20 ms limit
    assert elapsed[1] < 1e9                    # left through the abort flag, not its 1.4 s limit
    assert apb.device_status(ws, clear=True) == apb.APB_ERR_TIMEOUT
    assert apb.device_status(ws) == apb.APB_OK

    # the context is still usable: a normal prefill on the same workspace
    cfg = inputs.TINY
    x = inputs.generate(cfg)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    c = apb.make_config(cfg)
    run = apb.Prefill(c)
    run.workspace = torch.zeros_like(run.workspace)
    out = run(xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"], xd["b2"])
    torch.cuda.synchronize()
    assert apb.device_status(run.workspace) == apb.APB_OK
    assert torch.isfinite(out.float()).all()

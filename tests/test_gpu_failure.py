"""Failure detection on the GPU without a fault: a bounded wait that runs out,
and kernels whose waits are made to run out mid-run by a short wait limit.

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



@pytest.mark.gpu
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


@pytest.mark.gpu
@pytest.mark.parametrize("limit_ns", [2_000, 200])
def test_short_wait_limit_mid_kernel_is_reported_and_context_survives(limit_ns):
    """With the bounded waits' limit cut to microseconds, the waits that
    really block (on the tensor core, the copies, the other warps) run out
    mid-run in the score and attention kernels.  Each call must still finish
    -- every warp drains and meets its partners at each remaining named
    barrier -- and report APB_ERR_TIMEOUT; with the limit restored, the next
    run equals a clean run made before."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_apb_b200 import _lib as apb

    cfg = inputs.LLAMA8B_32K
    x = inputs.generate(cfg)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    c = apb.make_config(cfg)
    w = (xd["w1"], xd["b1"], xd["w2"], xd["b2"])
    run = apb.Prefill(c)
    ref = run(xd["q"], xd["k"], xd["v"], *w).clone()
    torch.cuda.synchronize()
    assert apb.device_status(run.workspace) == apb.APB_OK
    ws = run.workspace
    try:
        apb.selftest_set_wait_limit(limit_ns)
        apb.block_attention(c, xd["q"], xd["k"], xd["v"], run.pass_k, run.pass_v, out=run.out,
                            workspace=ws)
        torch.cuda.synchronize()
        assert apb.device_status(ws, clear=True) == apb.APB_ERR_TIMEOUT
        apb.score_compress(c, xd["q"], xd["k"], xd["v"], *w, idx=run.idx, workspace=ws)
        torch.cuda.synchronize()
        assert apb.device_status(ws, clear=True) == apb.APB_ERR_TIMEOUT
    finally:
        apb.selftest_set_wait_limit(0)
    out = run(xd["q"], xd["k"], xd["v"], *w)
    torch.cuda.synchronize()
    assert apb.device_status(ws) == apb.APB_OK
    assert torch.equal(out, ref)


def test_wait_limit_argument_checks():
    from long_context_sparse_apb_b200 import _lib as apb
    assert apb._lib.apb_selftest_set_wait_limit(50) == apb.APB_ERR_INVALID_ARG
    assert "limit_ns=50" in apb._lib.apb_last_error().decode()
    assert apb._lib.apb_selftest_set_wait_limit(0) == apb.APB_OK

"""Failure detection on the GPU without a fault: a bounded wait that runs out,
and kernels whose waits are made to give up mid-run through the launch-wide
abort flag.

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


def test_abort_mid_kernel_is_reported_and_context_survives():
    """A kernel whose waits start giving up mid-run (the launch-wide abort
    flag set from another stream, as a CTA whose wait ran out would set it)
    must still finish -- every warp meets its partners at each remaining
    named barrier -- and report APB_ERR_TIMEOUT; the context stays usable
    and the next clean run equals a clean run made before."""
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
    side = torch.cuda.Stream()

    # attention (~2 ms at 32K): the one-thread abort kernel fits beside the
    # attention CTAs and fires 0.5 ms into the launch
    ws = run.workspace
    ws.zero_()
    torch.cuda.synchronize()
    apb.block_attention(c, xd["q"], xd["k"], xd["v"], run.pass_k, run.pass_v, out=run.out,
                        workspace=ws)
    apb.selftest_abort_after(ws, 500, stream=side)
    torch.cuda.synchronize()
    assert apb.device_status(ws, clear=True) == apb.APB_ERR_TIMEOUT

    ws.zero_()
    out = run(xd["q"], xd["k"], xd["v"], *w)
    torch.cuda.synchronize()
    assert apb.device_status(ws) == apb.APB_OK
    assert torch.equal(out, ref)


def test_abort_mid_score_kernel_is_reported():
    """The same for the persistent score kernel (128K workload, ~0.5 ms):
    the abort kernel goes first (it holds one SM, so one CTA pair starts only
    after it and leaves at once) and fires 0.25 ms later, well after the
    call's own clearing of the flag and inside the score kernel."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_apb_b200 import _lib as apb

    cfg = inputs.LLAMA8B_128K
    x = inputs.generate(cfg)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    del x
    c = apb.make_config(cfg)
    w = (xd["w1"], xd["b1"], xd["w2"], xd["b2"])
    ws = apb.new_workspace(c)
    ref, _ = apb.score_compress(c, xd["q"], xd["k"], xd["v"], *w, workspace=ws)
    torch.cuda.synchronize()
    assert apb.device_status(ws) == apb.APB_OK
    side = torch.cuda.Stream()
    ws.zero_()
    torch.cuda.synchronize()
    apb.selftest_abort_after(ws, 250, stream=side)
    apb.score_compress(c, xd["q"], xd["k"], xd["v"], *w, workspace=ws)
    torch.cuda.synchronize()
    assert apb.device_status(ws, clear=True) == apb.APB_ERR_TIMEOUT
    ws.zero_()
    idx, _ = apb.score_compress(c, xd["q"], xd["k"], xd["v"], *w, workspace=ws)
    torch.cuda.synchronize()
    assert apb.device_status(ws) == apb.APB_OK
    assert torch.equal(idx, ref)

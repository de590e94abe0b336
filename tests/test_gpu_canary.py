"""Out-of-range writes (compute-sanitizer is not available): every output of
every C-ABI call is a view into a larger buffer whose guard regions before
and after it are filled with a canary pattern; after the calls on ragged
shapes (n and keep not multiples of the 128-row tile, G = 5, d = 64 and 128)
the guards must be untouched, and the outputs themselves fully written."""
import pytest
import torch

from long_context_sparse_apb_b200 import inputs

pytestmark = pytest.mark.gpu

GUARD = 4096                  # bytes on each side (a multiple of 16: keeps the view aligned)
CANARY = 0x5A


@pytest.fixture(scope="module")
def apb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_apb_b200 import _lib
    return _lib


class Guarded:
    """A tensor of `shape`/`dtype` inside a canary-filled byte buffer."""

    def __init__(self, shape, dtype):
        n = 1
        for s in shape:
            n *= s
        self.nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.buf = torch.full((GUARD + self.nbytes + GUARD,), CANARY, dtype=torch.uint8,
                              device="cuda")
        self.t = self.buf[GUARD:GUARD + self.nbytes].view(dtype).view(shape)

    def guards_intact(self):
        return bool((self.buf[:GUARD] == CANARY).all()) and \
            bool((self.buf[GUARD + self.nbytes:] == CANARY).all())

    def fully_written(self):
        # the canary byte pattern cannot survive in every byte of a written
        # region of this size unless the kernel skipped it
        body = self.buf[GUARD:GUARD + self.nbytes]
        return not bool((body == CANARY).all())


SHAPES = [
    inputs.TINY.replace(n_hosts=3, block_len=300, anchor_len=75, keep=130, n_q_heads=10,
                        n_kv_heads=2, head_dim=128, seed=31),
    inputs.TINY.replace(n_hosts=2, block_len=257, anchor_len=64, keep=1, n_q_heads=4,
                        n_kv_heads=4, head_dim=64, seed=32),
]


@pytest.mark.parametrize("cfg", SHAPES, ids=["ragged_d128_g5", "ragged_d64_keep1"])
def test_outputs_stay_inside_their_buffers(apb, cfg):
    x = inputs.generate(cfg)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    c = apb.make_config(cfg)
    N, hq, hkv, d, H, keep = cfg.seq_len, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, \
        cfg.n_hosts, cfg.keep
    w = (xd["w1"], xd["b1"], xd["w2"], xd["b2"])
    scores = Guarded((hkv, N), torch.float32)
    idx = Guarded((H, hkv, keep), torch.int32)
    pk = Guarded((H * keep, hkv, d), torch.bfloat16)
    pv = Guarded((H * keep, hkv, d), torch.bfloat16)
    out = Guarded((N, hq, d), torch.bfloat16)
    lse = Guarded((hq, N), torch.float32)
    ws = apb.new_workspace(c)

    apb.score_compress(c, xd["q"], xd["k"], xd["v"], *w, scores=scores.t, idx=idx.t, workspace=ws)
    apb.build_passing(c, xd["k"], xd["v"], idx.t, pk.t, pv.t)
    apb.block_attention(c, xd["q"], xd["k"], xd["v"], pk.t, pv.t, out=out.t, lse=lse.t,
                        workspace=ws)
    torch.cuda.synchronize()
    assert apb.device_status(ws) == apb.APB_OK
    for name, g in (("scores", scores), ("idx", idx), ("pass_k", pk), ("pass_v", pv),
                    ("out", out), ("lse", lse)):
        assert g.guards_intact(), name
        assert g.fully_written(), name

    # the fused compression and the one-call prefill into fresh guarded buffers
    idx2 = Guarded((H, hkv, keep), torch.int32)
    pk2 = Guarded((H * keep, hkv, d), torch.bfloat16)
    pv2 = Guarded((H * keep, hkv, d), torch.bfloat16)
    apb.score_compress_pass(c, xd["q"], xd["k"], xd["v"], *w, pk2.t, pv2.t, idx=idx2.t,
                            workspace=ws)
    out2 = Guarded((N, hq, d), torch.bfloat16)
    lse2 = Guarded((hq, N), torch.float32)
    pws = Guarded((apb.prefill_workspace_bytes(c),), torch.uint8)
    pws.t.zero_()
    apb.prefill(c, xd["q"], xd["k"], xd["v"], *w, out=out2.t, lse=lse2.t, workspace=pws.t)
    torch.cuda.synchronize()
    assert apb.device_status(pws.t) == apb.APB_OK
    for name, g in (("idx (fused)", idx2), ("pass_k (fused)", pk2), ("pass_v (fused)", pv2),
                    ("out (prefill)", out2), ("lse (prefill)", lse2), ("prefill workspace", pws)):
        assert g.guards_intact(), name
    assert torch.equal(idx2.t, idx.t)
    assert torch.equal(pk2.t.view(torch.int16), pk.t.view(torch.int16))
    assert torch.equal(pv2.t.view(torch.int16), pv.t.view(torch.int16))
    assert torch.equal(out2.t, out.t) and torch.equal(lse2.t, lse.t)

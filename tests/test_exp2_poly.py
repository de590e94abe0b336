"""Error bound of the FMA-pipe 2^x used for a share of the softmax
probabilities (exp2_poly2 in csrc/sm100_ptx.cuh), emulated step by step in
float32 with the constants read from the header: magic-number rounding,
f = x - n, degree-3 polynomial, exponent-field add.  The bf16 probabilities
it feeds are rounded to 2^-9 relative, so the bound asked here is 1e-4."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "long_context_sparse_apb_b200", "csrc", "sm100_ptx.cuh")


def _consts():
    text = open(HDR).read()
    body = text[text.index("exp2_poly2"):]
    c = dict(re.findall(r"\b(c[0-3]) = ([0-9.]+)f", body))
    magic = float(re.search(r"kMagic = ([0-9.]+)f", body).group(1))
    return [np.float32(c[f"c{i}"]) for i in range(4)], np.float32(magic)


def _emulate(x):
    (c0, c1, c2, c3), magic = _consts()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (n * np.float32(-1.0) + x).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-124.0, 9.0, 2_000_001, dtype=np.float32)
    y = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_masked_and_tiny_inputs_stay_tiny_positive():
    y = _emulate(np.array([-np.inf, -1e30, -200.0, -125.0], dtype=np.float32))
    assert np.all(y > 0) and np.all(y < 1e-37)

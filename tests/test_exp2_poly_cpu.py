"""The polynomial 2^f the forward kernel uses for part of its exponentials:
its coefficients (read from the kernel source) must be a near-minimax
relative-error fit of 2^f on [-1/2, 1/2] (bound 7.5e-5), and continuous
across the integer split (p(1/2) = 2 p(-1/2) to within that bound)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def coefficients():
    src = open(os.path.join(ROOT, "exact_attention_156_b200", "csrc", "ptx.cuh")).read()
    body = src[src.index("f2_exp2_poly(uint64_t x)"):]
    body = body[:body.index("f2_unpack(q, q0, q1)")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)]
    c3, c2, c1, c0 = vals[-4:]  # after the rounding constant
    return c0, c1, c2, c3


def test_polynomial_error_bound():
    c0, c1, c2, c3 = coefficients()
    f = np.linspace(-0.5, 0.5, 200001)
    p = ((c3 * f + c2) * f + c1) * f + c0
    rel = np.abs(p - 2.0 ** f) / 2.0 ** f
    assert rel.max() < 7.6e-5
    # equioscillation: the error reaches its bound with both signs
    e = (p - 2.0 ** f) / 2.0 ** f
    assert e.max() > 7.0e-5 and e.min() < -7.0e-5


def test_float32_split_reproduces_exp2():
    c0, c1, c2, c3 = (np.float32(c) for c in coefficients())
    x = np.random.default_rng(0).uniform(-126, 127, 200000).astype(np.float32)
    magic = np.float32(12582912.0)
    j = (np.maximum(x, np.float32(-126)) + magic).astype(np.float32)
    n = (j - magic).astype(np.float32)
    fr = (x - n).astype(np.float32)
    q = (((c3 * fr + c2) * fr + c1) * fr + c0).astype(np.float32)
    bits = q.view(np.int32) + (j.view(np.int32) << 23)
    y = bits.view(np.float32).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y - ref) / ref) < 8e-5

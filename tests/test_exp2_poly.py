"""The polynomial exp2 of the prefill softmax: constants and error bound.

The kernel computes 2^x on the FMA pipe for part of the softmax as 2^n * p(f), with
n = round(x) (obtained by adding and subtracting 1.5*2^23), f = x - n and p the degree-3
relative-minimax polynomial of 2^f on [-1/2, 1/2].  This test reads the constants from the
kernel source, checks them against the Remez generator that lives beside the kernel, and
replays the same float32 steps in numpy over the kernel's input range to bound the error.
"""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "long_context_prefill_estimate_b200", "csrc")


def _kernel_constants():
    src = open(os.path.join(CSRC, "rr_prefill_tc.cu")).read()
    body = src[src.index("exp2_poly2(f32x2 x"):]
    body = body[: body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([-0-9.e+]+)f, \1f\)", body)]
    magic, neg_magic, minus1, c3, c2, c1, c0 = vals
    assert magic == 12582912.0 and neg_magic == -magic and minus1 == -1.0
    return np.float32([c0, c1, c2, c3])


def _poly_exp2(x):
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    nf = (t - magic).astype(np.float32)
    f = (x - nf).astype(np.float32)
    c0, c1, c2, c3 = _kernel_constants()
    q = (c3 * f + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_constants_match_the_generator():
    sys.path.insert(0, CSRC)
    try:
        import gen_exp2_poly
    finally:
        sys.path.pop(0)
    c, err = gen_exp2_poly.remez_exp2(3)
    np.testing.assert_allclose(_kernel_constants(), np.float32(c), rtol=1e-6)
    assert err < 1e-4


def test_relative_error_over_the_softmax_range():
    # softmax inputs are s*scale - max <= 8 (lazily rescaled max); results are normal floats
    # for x >= -125
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), -np.logspace(-8, 2, 10001),
                        np.arange(-125, 9, dtype=np.float64)]).astype(np.float32)
    got = _poly_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1.2e-4, rel.max()


def test_underflow_is_tiny_and_positive():
    x = np.float32([-125.5, -126.0, -126.5, -127.0, -150.0, -1e4, -np.inf])
    got = _poly_exp2(x)
    assert np.all(np.isfinite(got)) and np.all(got > 0) and np.all(got < 2.0 ** -124)

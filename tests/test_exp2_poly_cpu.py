"""The tensor-core softmax evaluates one exp2 pair in four on the FMA pipe
(exp2_poly2 in attn_tc.cu).  This replays its float32 arithmetic in numpy with
the coefficients read from the kernel source and checks it against the exact
2^x: relative error below 4e-6 over the range the softmax uses, exact at
integers' neighbourhood of 1, and no NaN/Inf for inputs clamped at -126."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs():
    src = open(os.path.join(ROOT, "lossless_diffusion_speculative_b200", "csrc", "attn_tc.cu")).read()
    body = src[src.index("float2 exp2_poly2(float2 x)"):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"make_float2\(([0-9.eE+-]+)f, \1f\)", body)]
    assert len(vals) == 5, vals
    return [np.float32(v) for v in vals]        # c4, c3, c2, c1, c0 in Horner order


def _fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def poly_exp2(x):
    c4, c3, c2, c1, c0 = _coeffs()
    x = np.maximum(np.float32(x), np.float32(-126.0)).astype(np.float32)
    k = np.float32(12582912.0)
    t = (x + k).astype(np.float32)
    n = (t - k).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = _fma32(c4, f, c3)
    q = _fma32(q, f, c2)
    q = _fma32(q, f, c1)
    q = _fma32(q, f, c0)
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_softmax_range():
    x = np.linspace(-120.0, 8.0, 400001).astype(np.float32)
    got = poly_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 4e-6, rel.max()


def test_near_zero_and_integers():
    x = np.array([0.0, -1.0, -2.0, 1.0, 8.0, -0.5, 0.5, -1e-7], np.float32)
    got = poly_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert (np.abs(got - ref) / ref).max() < 4e-6


def test_clamped_inputs_stay_finite_and_tiny():
    x = np.array([-126.0, -200.0, -1e30], np.float32)
    got = poly_exp2(x)
    assert np.isfinite(got).all() and (got >= 0).all() and (got < 2e-38).all()

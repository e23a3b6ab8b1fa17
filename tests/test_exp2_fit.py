"""Derivation of the polynomial exp2 the softmax runs on the FMA pipe.

The kernel evaluates 2^x for some score pairs as 2^n * p(f), n = round(x),
f = x - n in [-1/2, 1/2], with p(f) = 1 + c1 f + c2 f^2 + c3 f^3 (p(0) = 1 so
integer arguments are exact).  c1..c3 are the minimax fit of the relative
error on [-1/2, 1/2]; this test re-derives them with Lawson's iteratively
reweighted least squares (the weights converge to the minimax solution) and
checks the constants in csrc/sm100_ptx.cuh against the result and against
the stated bound.  The GPU test compares the compiled routine with exp2f.
"""

import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "kv_cache_reuse_falcon_b200", "csrc", "sm100_ptx.cuh")


def source_coefficients():
    text = open(SRC).read()
    vals = {}
    for name in ("kC1", "kC2", "kC3"):
        m = re.search(r"%s\s*=\s*(0x[0-9a-fA-Fp.+-]+)f;" % name, text)
        assert m, name
        vals[name] = float.fromhex(m.group(1))
    return np.array([vals["kC1"], vals["kC2"], vals["kC3"]])


def lawson_fit(iters=600, npts=4001):
    f = np.linspace(-0.5, 0.5, npts)
    y = np.exp2(f)
    A = np.stack([f, f ** 2, f ** 3], 1) / y[:, None]   # relative error of p: (A c - b)
    b = (y - 1.0) / y
    w = np.full(npts, 1.0 / npts)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        e = np.abs(A @ c - b)
        w = w * e
        w /= w.sum()
    return c


def max_rel_error(c, npts=200001):
    f = np.linspace(-0.5, 0.5, npts)
    p = 1.0 + f * (c[0] + f * (c[1] + f * c[2]))
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


def test_coefficients_are_the_minimax_relative_fit():
    c_src = source_coefficients()
    c_fit = lawson_fit()
    assert np.allclose(c_src, c_fit, rtol=2e-6, atol=0), (c_src, c_fit)
    # equioscillation: the error of the fit is no larger than the fitted one
    assert max_rel_error(c_src) <= 1.02e-4
    assert abs(max_rel_error(c_src) - max_rel_error(c_fit)) < 1e-7


def test_fp32_evaluation_path_against_exp2():
    """The kernel's float32 steps (clamp, round by 1.5*2^23, Horner, exponent add), emulated."""
    c1, c2, c3 = (np.float32(v) for v in source_coefficients())
    x = np.concatenate([np.linspace(-126.0, 8.0, 400001, dtype=np.float32),
                        np.arange(-120, 9, dtype=np.float32)])
    magic = np.float32(12582912.0)
    xc = np.maximum(x, np.float32(-127.0))
    t = (xc + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    fr = (xc - n).astype(np.float32)

    def fma(a, b, c):   # one rounding: the float64 product of two float32 values is exact
        return (a.astype(np.float64) * b + c).astype(np.float32)

    p = fma(np.full_like(fr, c3), fr, np.full_like(fr, c2))
    p = fma(p, fr, np.full_like(fr, c1))
    p = fma(p, fr, np.ones_like(fr))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    y = bits.view(np.float32).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1.0)) < 1.2e-4
    ints = np.arange(-120, 9, dtype=np.float32)
    k = np.searchsorted(x[-len(ints):], ints) + len(x) - len(ints)
    assert np.array_equal(y[k], np.exp2(ints.astype(np.float64)))

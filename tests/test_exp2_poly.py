"""The FMA-pipe exponential of the attention and group-scores kernels, checked on the CPU.

The kernel computes 2^x for x <= 1/2 as: clamp at -126, split x = n + f with
n = rint(x) through the 1.5*2^23 shift, a degree-5 polynomial p(f) ~ 2^f on
[-1/2, 1/2], and n added to p's exponent bits; results below 2^-126 are 0.
This test reads the coefficients out of the kernel source, replays those
steps bit for bit in float32 (numpy; fused multiply-adds through float64,
which is exact for a float32 product plus addend before the final rounding),
and compares with 2^x in float64.  It also re-derives the coefficients with
the fitting script and checks they agree with the ones in the kernel.
"""
import os
import re

import numpy as np

from sparse_attention_diffusion_mcs_b200 import fit_exp2_poly

SRC = os.path.join(os.path.dirname(__file__), "..", "sparse_attention_diffusion_mcs_b200", "csrc",
                   "mcs_common.cuh")


def _kernel_coeffs():
    body = open(SRC).read()
    fn = body[body.index("float ex2_fma(float x)"):]
    fn = fn[:fn.index("\n}\n")]
    nums = [float(v) for v in re.findall(r"([0-9]\.[0-9]+e[-+][0-9]+)f", fn)]
    # Horner order in the source: c5, c4, c3, c2, c1, c0
    assert len(nums) == 6, nums
    return np.array(nums[::-1], dtype=np.float32)   # c0..c5


def _fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def ex2_fma_emulated(x, c):
    x = np.float32(x)
    xc = np.float32(max(x, np.float32(-126.0)))
    y = np.float32(xc + np.float32(12582912.0))
    f = np.float32(xc - np.float32(y - np.float32(12582912.0)))
    p = _fma32(c[5], f, c[4])
    for ci in (c[3], c[2], c[1], c[0]):
        p = _fma32(p, f, ci)
    r = (np.array(p, np.float32).view(np.uint32) + (np.array(y, np.float32).view(np.uint32) << np.uint32(23)))
    return np.float32(r.astype(np.uint32).view(np.float32)) if x >= -126.0 else np.float32(0.0)


def test_kernel_coefficients_are_the_fitted_ones():
    c_fit, err = fit_exp2_poly.remez()
    assert err < 1e-7
    np.testing.assert_allclose(_kernel_coeffs(), np.float32(c_fit), rtol=1e-6)


def test_ex2_fma_matches_exp2_over_the_range():
    c = _kernel_coeffs()
    rng = np.random.default_rng(7)
    xs = np.concatenate([rng.uniform(-125.9, 0.5, 20000), rng.uniform(-3, 0.5, 20000),
                         np.arange(-126, 1, dtype=np.float64),           # exact integers: f = 0
                         np.arange(-126, 0) + 0.5,                         # ties of the split
                         [0.5, -0.5, -1e-30, 0.0]]).astype(np.float32)
    got = np.array([ex2_fma_emulated(x, c) for x in xs], dtype=np.float64)
    ref = np.exp2(xs.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 4e-7, (xs[np.argmax(rel)], rel.max())


def test_ex2_fma_flushes_below_the_normal_range():
    c = _kernel_coeffs()
    for x in [-126.0001, -127.0, -150.0, -1e30, -np.inf]:
        assert ex2_fma_emulated(np.float32(x), c) == 0.0
    smallest = float(ex2_fma_emulated(np.float32(-126.0), c))   # p(0) = c0, one ulp above 1
    assert abs(smallest - 2.0 ** -126) <= 4e-7 * 2.0 ** -126

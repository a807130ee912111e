"""The FMA-pipe 2^x of the forward kernel (csrc/sm100.cuh, ex2_poly2) against its error
bound. The constants are read from the kernel source and the kernel's float32 steps
(clamp, 1.5 * 2^23 shift, Horner, exponent add) are replayed bit for bit in numpy."""
import os
import re

import numpy as np

from piecewise_attention_diffusion_b200 import exp2_poly_fit

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "piecewise_attention_diffusion_b200", "csrc", "sm100.cuh")
BOUND = 8e-5  # relative; far below bf16's unit roundoff 2^-8 ~ 3.9e-3


def _kernel_constants():
    src = open(SRC).read()
    vals = {k: float(v) for k, v in re.findall(r"kEx2C([0-3]) = ([0-9.eE+-]+)f", src)}
    assert sorted(vals) == ["0", "1", "2", "3"]
    body = src[src.index("float2 ex2_poly2(float2 x)"):]
    body = body[:body.index("\n}\n")]
    # Horner order in the kernel: c3 * f + c2, then * f + c1, then * f + c0
    assert body.index("kEx2C3") < body.index("kEx2C1") < body.index("kEx2C0")
    return [np.float32(vals[str(i)]) for i in range(4)]


def _ex2_poly(x):
    """The kernel's float32 steps, lane by lane (f32x2 lanes round like scalar ops)."""
    f32 = np.float32
    c0, c1, c2, c3 = _kernel_constants()
    x = np.maximum(x.astype(f32), f32(-126.0))
    t = (x + f32(12582912.0)).astype(f32)
    f = (x - (t - f32(12582912.0)).astype(f32)).astype(f32)
    fma = lambda a, b, c: (a.astype(np.float64) * b + c).astype(f32)  # one rounding
    p = fma(f, c3, c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    n = (t.view(np.int32) - np.int32(0x4B400000)).astype(np.uint32)
    shifted = t.view(np.uint32) << np.uint32(23)   # what the kernel adds
    np.testing.assert_array_equal(shifted, n << np.uint32(23))
    return (p.view(np.uint32) + shifted).view(f32)


def test_constants_match_the_fit():
    c, err = exp2_poly_fit.remez_exp2(3)
    assert err < BOUND
    np.testing.assert_array_equal(np.asarray(_kernel_constants()), c.astype(np.float32))


def test_relative_error_bound_over_the_used_range():
    x = np.concatenate([np.linspace(-126.0, 16.0, 2_000_001),
                        np.random.default_rng(0).uniform(-30, 16, 1_000_000)]).astype(np.float32)
    got = _ex2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    normal = want >= 2.0 ** -125
    rel = np.abs(got[normal] - want[normal]) / want[normal]
    assert rel.max() < BOUND
    # integers are exact up to the polynomial's value at 0
    xi = np.arange(-120, 17).astype(np.float32)
    np.testing.assert_allclose(_ex2_poly(xi), np.exp2(xi.astype(np.float64)), rtol=1e-4)
    # below the clamp the result is a tiny positive number, never negative or NaN
    tiny = _ex2_poly(np.asarray([-1e30, -200.0, -126.7], dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 2.0 ** -120) and np.isfinite(tiny).all()

"""The attention kernel evaluates an eighth of its exponentials with a cubic
on the FMA pipe (exp2_poly in csrc/tt_attn.cu).  This re-evaluates that
routine in float32 with the coefficients read from the kernel source and
checks it against the exact 2^x: relative error below 1e-4 (P is then
rounded to bf16, whose relative spacing is 2^-8), exact powers of two at
integers, and 0 at or below -126."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_wise_diffusion_b200", "csrc", "tt_attn.cu")


def _coeffs():
    body = open(SRC).read().split("float exp2_poly(float x)")[1].split("\n}")[0]
    # the polynomial is the fmaf nest fmaf(fmaf(fmaf(c3, f, c2), f, c1), f, c0)
    nest = body[body.index("fmaf("):]
    nums = [float(v) for v in re.findall(r"(-?\d+\.\d+)f", nest)]
    c3, c2, c1, c0 = nums[:4]
    magic = [float(v) for v in re.findall(r"(\d+\.\d+)f", body[:body.index("fmaf(")])]
    assert magic == [126.0, 12582912.0, 12582912.0], magic
    return c0, c1, c2, c3


def exp2_poly(x):
    """float32 re-evaluation of the kernel routine, step by step."""
    c0, c1, c2, c3 = (np.float32(v) for v in _coeffs())
    magic = np.float32(12582912.0)              # 1.5 * 2^23
    x = np.asarray(x, np.float32)
    xc = np.maximum(x, np.float32(-126.0))
    t = (xc + magic).astype(np.float32)         # round-to-nearest-even integer in the low bits
    f = (xc - (t - magic)).astype(np.float32)
    p = (((c3 * f + c2) * f + c1) * f + c0).astype(np.float32)
    e = (t.view(np.int32) - np.int32(0x4B400000)) << 23
    r = (p.view(np.int32) + e).view(np.float32)
    return np.where(x > -126.0, r, np.float32(0.0))


def test_exp2_poly_reduction_is_round_to_nearest():
    x = np.float32([-2.5, -0.5, 0.49, 0.5, 1.5, 3.75, -125.2])
    xc = np.maximum(x, np.float32(-126.0))
    t = (xc + np.float32(12582912.0)).astype(np.float32)
    n = t.view(np.int32) - np.int32(0x4B400000)
    np.testing.assert_array_equal(n, np.rint(x).astype(np.int32))


def test_exp2_poly_relative_error():
    x = np.concatenate([np.linspace(-125.9, 8.0, 400001), -np.logspace(-6, 2, 1000)]).astype(np.float32)
    got = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1)) < 1e-4


def test_exp2_poly_integers_and_underflow():
    for n in range(-125, 9):
        assert abs(float(exp2_poly(np.float32(n))) / 2.0 ** n - 1) < 1e-4
    assert float(exp2_poly(np.float32(-126.0))) == 0.0
    assert float(exp2_poly(np.float32(-1e30))) == 0.0
    assert float(exp2_poly(np.float32(-np.inf))) == 0.0

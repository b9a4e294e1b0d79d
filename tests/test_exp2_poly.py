"""Pin of the FMA-pipe exp2 the attention softmax uses for part of its
columns: the coefficients exactly as written in the kernel source, evaluated
with the kernel's fp32 steps (round-to-nearest split by the 1.5*2^23 shift,
Horner, exponent-field add), must stay within a relative error of 1e-4 of
2^x over the range the softmax feeds it (x in [-125, 8]; smaller x is
clamped to -125, giving 2^-125, which vanishes against a row sum >= 1); far
below the 2^-8 relative spacing of the bf16 probabilities it produces."""
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "joint_video_audio_rope_b200", "csrc")


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "common.cuh")).read()
    body = src[src.index("exp2_poly_f32x2(uint64_t x2"):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"pack_f32x2\(([0-9.e-]+)f, \1f\)", body)]
    # shift constants first, then the Horner order c3, c2, c1, c0
    assert vals[:3] == [12582912.0, -12582912.0, -1.0], vals
    vals = vals[3:]
    assert len(vals) == 4, vals
    return np.array(vals[::-1], np.float32)


def _eval(c, x):
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = c[3]
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    return (p.view(np.int32) + (t.view(np.int32) << 23)).astype(np.int32).view(np.float32)


def test_kernel_exp2_polynomial_error_bound():
    c = _kernel_coefficients()
    x = np.concatenate([np.linspace(-125.0, 8.0, 1_000_001),
                        np.arange(-125, 8, dtype=np.float64) + 0.5,  # rounding ties
                        np.arange(-125, 9, dtype=np.float64)]).astype(np.float32)
    got = _eval(c, x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()
    assert np.all(got > 0) and np.all(np.isfinite(got))
    tiny = _eval(c, np.array([-126.0, -300.0, -np.inf], np.float32))
    assert np.all(tiny > 0) and np.all(tiny < 2.0 ** -124)


def test_exponent_trick_identity():
    # bits(t) << 23 == j << 23 (mod 2^32) for t = j + 1.5 * 2^23
    for j in range(-125, 9):
        t = np.float32(j) + np.float32(12582912.0)
        lhs = (int(np.array(t, np.float32).view(np.int32)) << 23) & 0xFFFFFFFF
        rhs = (j << 23) & 0xFFFFFFFF
        assert lhs == rhs

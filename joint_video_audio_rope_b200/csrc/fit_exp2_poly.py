"""Fit the polynomial of the FMA-pipe exp2 used by the attention softmax.

The kernel computes 2^x for x <= 8 as 2^j * 2^f with j = round(x) and
f = x - j in [-1/2, 1/2] (range reduction after Cody and Waite, "Software
Manual for the Elementary Functions", 1980), and 2^f by a degree-3
polynomial evaluated in fp32 with Horner's rule.  This script derives the
coefficients by a weighted least-squares fit of the relative error on a
dense grid, refined by iteratively reweighted least squares (Lawson's
algorithm) towards the minimax solution, rounds them to fp32, and prints the
resulting worst relative error (evaluated in float32 arithmetic, the
precision the kernel uses).

    python joint_video_audio_rope_b200/csrc/fit_exp2_poly.py

The probabilities this feeds are rounded to bf16 (relative spacing 2^-8), so
a relative error around 1e-4 is far below what the rounding already costs.
"""
import numpy as np


def fit(degree: int = 3, iters: int = 200):
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative error
    w = np.ones_like(f)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(A * w[:, None], w, rcond=None)
        err = np.abs(A @ c - 1.0)
        w = w * (err + 1e-18) ** 0.5
        w /= w.max()
    return c


def eval_f32(c, x):
    """The kernel's arithmetic on float32: round-to-nearest split, Horner."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    fr = (x - j).astype(np.float32)
    c32 = c.astype(np.float32)
    p = c32[3]
    for k in (2, 1, 0):
        p = (p * fr + c32[k]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    x = np.linspace(-125.0, 8.0, 2_000_001).astype(np.float32)
    got = eval_f32(c32.astype(np.float64), x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.max(np.abs(got / ref - 1.0))
    for k, v in enumerate(c32):
        print(f"c{k} = {float(v)!r}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error on [-125, 8] in fp32: {rel:.3e}")

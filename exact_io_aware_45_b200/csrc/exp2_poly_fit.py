"""Derives the polynomial behind the forward kernel's FMA-pipe exp2.

2^x is split as 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2]
(Cody and Waite's range reduction, specialised to base 2); 2^f is then a
cubic in f. The cubic here is the least-squares fit of 2^f at 4096 Chebyshev
nodes on [-1/2, 1/2] under a relative-error weight, which is close to the
minimax cubic; its relative error (about 9e-5) is far below the 2^-9
rounding of the bf16 P it feeds.

    python exact_io_aware_45_b200/csrc/exp2_poly_fit.py

prints the four coefficients (c0 + c1 f + c2 f^2 + c3 f^3) as float32 and
the maximum relative error of the float32 evaluation, the numbers the kernel
source carries (kExp2P0..kExp2P3 in sm100_common.cuh).
"""
import numpy as np


def fit(degree: int = 3, nodes: int = 4096):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)          # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]   # relative-error weight
    c, *_ = np.linalg.lstsq(A, np.ones_like(f), rcond=None)
    return c.astype(np.float32)


def eval_f32(x, c):
    """The kernel's steps in float32: clamp x at -125, round x to j with the 1.5*2^23 shift,
    f = x - j, Horner cubic, then add j to the exponent field."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = c[3]
    for ci in (c[2], c[1], c[0]):
        p = (p * f + ci).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


if __name__ == "__main__":
    c = fit()
    print("coefficients:", ", ".join(f"{v:.9e}f" for v in c))
    x = np.linspace(-30.0, 8.0, 2_000_001, dtype=np.float32)
    rel = np.abs(eval_f32(x, c) / np.exp2(x.astype(np.float64)) - 1.0)
    print(f"max relative error on [-30, 8]: {rel.max():.3e}")

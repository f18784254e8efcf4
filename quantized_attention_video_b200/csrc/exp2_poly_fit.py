"""Fit the polynomial behind the FMA-pipe exp2 of the attention kernel.

2^u = 2^n * 2^r with n = rint(u), r = u - n in [-1/2, 1/2] (Cody-Waite style
range reduction).  2^r is approximated by a degree-5 polynomial fitted by least
squares on Chebyshev nodes in FP64 (a near-minimax fit of the relative error),
with c0 pinned to 1 so that 2^0 is exact.  The coefficients are rounded to FP32
and the relative error of the FP32 Horner evaluation (one rounding per fused
multiply-add) is measured on a dense grid against the exact 2^r.

    python exp2_poly_fit.py      # prints the coefficients and the error
"""
import numpy as np

DEG = 5


def fit(deg=DEG):
    k = np.arange(4000)
    r = 0.5 * np.cos(np.pi * (k + 0.5) / len(k))            # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(r)
    # relative-error weighting: minimise sum ((P(r) - 2^r) / 2^r)^2 with c0 = 1
    A = np.stack([r ** i for i in range(1, deg + 1)], axis=1) / y[:, None]
    b = (y - 1.0) / y
    c, *_ = np.linalg.lstsq(A, b, rcond=None)
    return np.concatenate([[1.0], c])


def horner_f32(c32, r):
    """FP32 Horner with one rounding per step (fma of FP32 operands is exact in FP64)."""
    p = np.full_like(r, c32[-1], dtype=np.float32)
    for ci in c32[-2::-1]:
        p = (p.astype(np.float64) * r.astype(np.float64) + np.float64(ci)).astype(np.float32)
    return p


def max_rel_error(c32):
    r = np.linspace(-0.5, 0.5, 2_000_001).astype(np.float32)
    p = horner_f32(c32, r).astype(np.float64)
    return float(np.max(np.abs(p / np.exp2(r.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci)!r}  ({np.float32(ci).view(np.uint32):#010x})")
    print("max relative error of the FP32 evaluation on [-1/2, 1/2]:", max_rel_error(c32))

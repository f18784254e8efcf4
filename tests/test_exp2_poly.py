"""The FMA-pipe exp2 of the attention kernel against the exact 2^u (an error bound).

Built with H3ATTN_FMA_EXP2_PAIRS_OF_8=k (k of every 8 key pairs; 0 by default,
where every probability comes from MUFU), the kernel evaluates part of its
probabilities without the MUFU unit: n = rint(u) through the 1.5*2^23 magic
number, r = u - n, 2^r by a degree-5 polynomial in FP32 Horner form (one
rounding per fused multiply-add), then n added into the exponent field.  This test reads the coefficients the kernel is
built with (csrc/exp2_poly.h), replays those exact FP32 steps in numpy and
checks the result against 2^u in FP64 over the argument range the kernel
produces (u in [-125, log2(448)]).  The bound it enforces, 2.5e-7 relative, is
that of the MUFU ex2.approx.f32 path the kernel uses for the other keys
(about 2^-22), with margin.
"""
import os
import re

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
HEADER = os.path.join(os.path.dirname(HERE), "quantized_attention_video_b200", "csrc", "exp2_poly.h")


def coefficients():
    text = open(HEADER).read()
    c = dict((int(i), np.float32(float(v))) for i, v in re.findall(r"kExp2C(\d)\s*=\s*([0-9.eE+-]+)f;", text))
    assert sorted(c) == list(range(6))
    return [c[i] for i in range(6)]


def fma32(a, b, c):
    # a*b of FP32 operands is exact in FP64; one rounding to FP32 after the add
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma(u):
    """Bit-level replay of exp2_fma_pair for FP32 arguments u."""
    u = np.maximum(u.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    y = (u + magic).astype(np.float32)                 # RN: magic + rint(u)
    n = (y - magic).astype(np.float32)                 # exact
    r = fma32(n, np.full_like(n, -1.0), u)              # u - n, exact
    c = coefficients()
    p = fma32(np.full_like(r, c[5]), r, np.full_like(r, c[4]))
    for ci in (c[3], c[2], c[1], c[0]):
        p = fma32(p, r, np.full_like(r, ci))
    bits = p.view(np.uint32).astype(np.uint64) + (y.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_coefficients_give_one_at_zero_and_log2_slope():
    c = coefficients()
    assert c[0] == np.float32(1.0)
    assert abs(float(c[1]) - np.log(2.0)) < 1e-6


def test_fma_exp2_relative_error_over_the_kernel_range():
    rng = np.random.default_rng(5)
    u = np.concatenate([
        np.linspace(-125.0, 8.8073549, 2_000_001),
        rng.uniform(-30.0, 8.8, 1_000_000),
        np.arange(-125, 9, dtype=np.float64),            # integers: r = 0
        np.arange(-125, 9, dtype=np.float64) + 0.5,      # ties of rint
    ]).astype(np.float32)
    got = exp2_fma(u).astype(np.float64)
    exact = np.exp2(np.maximum(u, -125.0).astype(np.float64))
    rel = np.abs(got / exact - 1.0)
    assert rel.max() < 2.5e-7, float(rel.max())
    assert np.all(got > 0) and np.all(np.isfinite(got))


def test_fma_exp2_clamps_far_below_the_max():
    u = np.array([-126.0, -200.0, -1e30], np.float32)
    got = exp2_fma(u)
    assert np.all(got > 0) and np.all(got < 2.0 ** -124)

"""Pins of the oracle's Q/K RMSNorm + RoPE (oracle.cpp, orc_qk_norm_rope).

The pages name the step ("H3 Performance Roadmap": "Norm and RoPE" in the
representative block table, and Component 2, item 1: Q/K normalization and RoPE
applied where the attention consumes Q and K) but give no formula; the oracle
takes a per-head RMSNorm r = 1/sqrt(mean(x^2) + eps), n = bf16(x r),
z = bf16(n gamma), then the rotation of channel pairs (2i, 2i+1) by the caller's
cos/sin table, rounded to BF16.  These tests check it against the FP64 formula
within a bound derived from its roundings, and against cases whose results are
exact (a rotation by 0 or by a quarter turn, a row whose norm is a power of two,
zero rows, scaling by powers of two).
"""
import numpy as np
import pytest

import oracle

D = 128


def _bf16(x):
    return oracle.bf16_encode(np.asarray(x, np.float32))


def _tables(T, rng):
    ang = rng.uniform(-np.pi, np.pi, size=(T, D // 2))
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def _fp64_reference(xb, gamma, eps, cos, sin):
    """x / sqrt(mean x^2 + eps) * gamma, then the pair rotation, all in FP64; also
    the unrotated normalized values (for the error bound)."""
    x = oracle.bf16_decode(xb).astype(np.float64)
    r = 1.0 / np.sqrt((x * x).mean(-1, keepdims=True) + eps)
    z = x * r * gamma.astype(np.float64)
    a, b = z[..., 0::2], z[..., 1::2]
    c = cos.astype(np.float64)[None, :, None, :]
    s = sin.astype(np.float64)[None, :, None, :]
    out = np.empty_like(z)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = b * c + a * s
    mag = np.empty_like(z)
    mag[..., 0::2] = np.abs(a * c) + np.abs(b * s)
    mag[..., 1::2] = np.abs(b * c) + np.abs(a * s)
    return out, mag


@pytest.mark.parametrize("eps", [1e-6, 0.5])
def test_against_fp64_formula_with_derived_bound(eps):
    # Bound: a BF16 rounding moves a value by at most 2^-8 of itself (half an ulp
    # of an 8-bit significand, relative to a value just above a power of two).
    # z carries two of them (n, then n*gamma) plus the FP32 roundings of the sum of
    # squares (12 in sequence, < 2^-20 relative) and of r (three, < 2^-22); the
    # rotation adds FP32 roundings (< 2^-22 of |a c| + |b s|)
    # and the final BF16 rounding.  So |out - ref| <= 2^-8 |ref| + 1.01 * 2^-7 *
    # (|a c| + |b s|).
    rng = np.random.default_rng(11)
    B, T, H = 2, 9, 3
    x = rng.standard_normal((B, T, H, D)) * rng.uniform(0.05, 4.0, size=(B, T, H, 1))
    xb = _bf16(x)
    gamma = oracle.bf16_decode(_bf16(rng.normal(1.0, 0.1, size=D))).astype(np.float32)
    cos, sin = _tables(T, rng)
    got = oracle.bf16_decode(oracle.qk_norm_rope(xb, gamma, eps, cos, sin)).astype(np.float64)
    ref, mag = _fp64_reference(xb, gamma, eps, cos, sin)
    bound = 2.0 ** -8 * np.abs(ref) + 1.01 * 2.0 ** -7 * mag + 1e-30
    assert np.all(np.abs(got - ref) <= bound), np.max(np.abs(got - ref) / bound)
    # the bound is tight enough to see a dropped gamma, a sum instead of a mean,
    # eps outside the square root, or rotate-half pairs (i, i + 64)
    for wrong in (
        _fp64_reference(xb, np.ones(D, np.float32), eps, cos, sin)[0],
        _fp64_reference(xb, gamma, eps, cos, sin)[0] / np.sqrt(D),
    ):
        assert np.any(np.abs(got - wrong) > bound)
    xf = oracle.bf16_decode(xb).astype(np.float64)
    z_out = xf / (np.sqrt((xf * xf).mean(-1, keepdims=True)) + eps) * gamma
    a, b = z_out[..., 0::2], z_out[..., 1::2]
    c, s = cos[None, :, None, :], sin[None, :, None, :]
    wrong = np.empty_like(z_out)
    wrong[..., 0::2], wrong[..., 1::2] = a * c - b * s, b * c + a * s
    if eps > 0.1:
        assert np.any(np.abs(got - wrong) > bound)
    zr = xf / np.sqrt((xf * xf).mean(-1, keepdims=True) + eps) * gamma
    lo, hi = zr[..., :64], zr[..., 64:]
    wrong = np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)
    assert np.any(np.abs(got - wrong) > bound)


def test_exact_norm_and_quarter_turns():
    # every channel +-1.5 and eps = 1.75: mean x^2 + eps = 4, r = 1/2 exactly, n = +-0.75,
    # gamma = 2 gives z = +-1.5; a rotation by 0 keeps z, by a quarter turn gives
    # (-z_2i+1, z_2i), by a half turn -z: all exact in BF16
    rng = np.random.default_rng(3)
    T, H = 3, 2
    signs = rng.choice([-1.0, 1.0], size=(1, T, H, D))
    xb = _bf16(1.5 * signs)
    gamma = np.full(D, 2.0, np.float32)
    cos = np.array([[1.0] * 64, [0.0] * 64, [-1.0] * 64], np.float32)
    sin = np.array([[0.0] * 64, [1.0] * 64, [0.0] * 64], np.float32)
    got = oracle.bf16_decode(oracle.qk_norm_rope(xb, gamma, 1.75, cos, sin))
    z = 1.5 * signs
    np.testing.assert_array_equal(got[:, 0], z[:, 0])
    quarter = np.empty_like(z[:, 1])
    quarter[..., 0::2], quarter[..., 1::2] = -z[:, 1, :, 1::2], z[:, 1, :, 0::2]
    np.testing.assert_array_equal(got[:, 1], quarter)
    np.testing.assert_array_equal(got[:, 2], -z[:, 2])


def test_zero_rows_stay_zero():
    xb = np.zeros((1, 4, 2, D), np.uint16)
    rng = np.random.default_rng(5)
    cos, sin = _tables(4, rng)
    got = oracle.bf16_decode(oracle.qk_norm_rope(xb, np.ones(D, np.float32), 1e-6, cos, sin))
    assert np.all(got == 0.0)


@pytest.mark.parametrize("k", [-6, 3])
def test_scaling_by_powers_of_two(k):
    # x -> 2^k x with eps -> 4^k eps scales mean + eps by 4^k, the square root by 2^k
    # and r by 2^-k, all exactly: the output bits are unchanged
    rng = np.random.default_rng(7 + k)
    T = 6
    x = rng.standard_normal((1, T, 2, D)).astype(np.float32)
    xb = _bf16(x)
    xs = _bf16(oracle.bf16_decode(xb) * np.float32(2.0 ** k))
    gamma = rng.normal(1.0, 0.1, size=D).astype(np.float32)
    cos, sin = _tables(T, rng)
    eps = 2.0 ** -10
    a = oracle.qk_norm_rope(xb, gamma, eps, cos, sin)
    b = oracle.qk_norm_rope(xs, gamma, eps * 4.0 ** k, cos, sin)
    np.testing.assert_array_equal(a, b)


def test_strided_views_and_heads_are_independent():
    # the packed [B, T, 3, H, D] layout read through a view gives the same rows as a
    # dense copy, and each head is normalized on its own channels only
    rng = np.random.default_rng(9)
    B, T, H = 1, 5, 3
    packed = _bf16(rng.standard_normal((B, T, 3, H, D)))
    cos, sin = _tables(T, rng)
    g = np.ones(D, np.float32)
    view = packed[:, :, 1]
    a = oracle.qk_norm_rope(view, g, 1e-6, cos, sin)
    b = oracle.qk_norm_rope(np.ascontiguousarray(view), g, 1e-6, cos, sin)
    np.testing.assert_array_equal(a, b)
    one = oracle.qk_norm_rope(np.ascontiguousarray(view[:, :, 1:2]), g, 1e-6, cos, sin)
    np.testing.assert_array_equal(a[:, :, 1:2], one)


def test_quantize_norm_rope_is_the_composition():
    rng = np.random.default_rng(13)
    B, T, H = 1, 70, 2
    q, k, v = (_bf16(rng.standard_normal((B, T, H, D))) for _ in range(3))
    cq, sq_ = _tables(T, rng)
    nr = dict(gamma_q=np.full(D, 1.25, np.float32), gamma_k=np.full(D, 0.75, np.float32), eps=1e-6,
              cos_q=cq, sin_q=sq_, cos_k=cq, sin_k=sq_)
    z = oracle.quantize_norm_rope(q, k, v, nr)
    qn = oracle.qk_norm_rope(q, nr["gamma_q"], 1e-6, cq, sq_)
    kn = oracle.qk_norm_rope(k, nr["gamma_k"], 1e-6, cq, sq_)
    z2 = oracle.quantize(qn, kn, v)
    for key in ("q8", "k8", "sq", "sk", "km", "v8", "sv"):
        np.testing.assert_array_equal(z[key], z2[key])
    # normalized rows have RMS about gamma: the Q scale groups see amax near 1.25 * 3..5
    assert 1.25 * 2.0 / 127 < float(z["sq"].max()) < 1.25 * 6.0 / 127


def test_rejects_bad_arguments():
    xb = np.zeros((1, 2, 1, D), np.uint16)
    c = np.ones((2, 64), np.float32)
    s = np.zeros((2, 64), np.float32)
    with pytest.raises(ValueError):
        oracle.qk_norm_rope(xb, np.ones(D, np.float32), 0.0, c, s)


def test_intermediate_roundings_golden():
    # Hand-derived values that fix the order of the roundings.  Every channel pair of the
    # row is (+1, -1): mean x^2 = 1; eps = 1.25 gives sqrt(2.25) = 1.5 exactly and
    # r = RN(1/1.5) = 0.666666686...; n = bf16(r) = 171/256 (the BF16 neighbours are 170/256
    # and 171/256; r lies above 170.67/256); gamma = 1.25: n*gamma = 855/1024 exactly, which
    # rounds to z = 214/256 = 0.8359375 (213.75/256).  Without rounding n first, r*1.25 =
    # 0.83333 rounds to 213/256 instead.
    #   token 0, cos 1, sin 0: out = (z, -z) = (0.8359375, -0.8359375).
    #   token 1, cos 0.625, sin 0.5: a*c - b*s = 214/256*5/8 + 214/256/2 = 1926/2048, which
    #   rounds to 241/256 = 0.94140625 (1926/8 = 240.75); b*c + a*s = -1070/2048 + 856/2048
    #   = -214/2048 = -0.1044921875 (exact in BF16).  Without rounding z first the first
    #   value is 7695/8192, which rounds to 240/256 = 0.9375.
    x = np.tile(np.array([1.0, -1.0], np.float32), 64).reshape(1, 1, 1, D)
    xb = _bf16(np.concatenate([x, x], axis=1))  # tokens 0 and 1
    gamma = np.full(D, 1.25, np.float32)
    cos = np.array([[1.0] * 64, [0.625] * 64], np.float32)
    sin = np.array([[0.0] * 64, [0.5] * 64], np.float32)
    got = oracle.bf16_decode(oracle.qk_norm_rope(xb, gamma, 1.25, cos, sin))
    np.testing.assert_array_equal(got[0, 0, 0], np.tile(np.array([0.8359375, -0.8359375], np.float32), 64))
    np.testing.assert_array_equal(got[0, 1, 0], np.tile(np.array([0.94140625, -0.1044921875], np.float32), 64))

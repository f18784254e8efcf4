"""Pins for the CPU oracle: each checks it against something other than itself.

Sources of truth used here: the FP8 E4M3 / bfloat16 casts of a library
(PyTorch CPU), integer matrix products (numpy int64), exact rational sums
(math.fsum), invariants the quantization policy implies, a closed form for a
permutation-one-hot V, an FP64 unquantized softmax attention with an error
bound derived from the arithmetic, and a hand-derived 4x4 case
(tests/golden/brute4x4.json).

The policy being pinned is that of the dense Sage-compatible attention:
"H3 Performance Roadmap", Phase 4: Dense Sage-Compatible Attention (per-warp
INT8 Q/K, FP8 V, K smoothing) and "Phase 2B Aligned Numerical Prototype",
Exactness (scores, per-epoch m and d, FP8 probability words, RO, reciprocal).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(x) -> np.ndarray:
    """float array -> BF16 bit patterns through PyTorch's cast (round to nearest even)."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_vals(bits) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).float().numpy()


E4M3_TORCH = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()


# ------------------------------------------------------------------ codecs --
def test_e4m3_decode_matches_library_table():
    tab = oracle.e4m3_decode_table()
    nan = np.isnan(E4M3_TORCH)
    assert np.array_equal(np.isnan(tab), nan)
    assert np.array_equal(tab[~nan], E4M3_TORCH[~nan])
    assert tab[0x7E] == 448.0 and tab[0x01] == 2.0 ** -9 and tab[0x08] == 2.0 ** -6


def test_e4m3_encode_roundtrip_and_midpoints():
    finite = [c for c in range(256) if not np.isnan(E4M3_TORCH[c])]
    vals = E4M3_TORCH[finite]
    enc = oracle.e4m3_encode(vals)
    # every representable value encodes to itself (the two zeros both decode to 0)
    assert np.array_equal(E4M3_TORCH[enc], vals)
    pos = np.sort(np.unique(vals[vals >= 0]))
    mids = (pos[:-1].astype(np.float64) + pos[1:]) / 2
    mids32 = mids.astype(np.float32)
    assert np.array_equal(mids32.astype(np.float64), mids)  # midpoints are exact in FP32
    got = E4M3_TORCH[oracle.e4m3_encode(mids32)]
    codes_lo = np.array([list(E4M3_TORCH).index(v) for v in pos[:-1]])
    # ties go to the even code (the code whose mantissa LSB is 0)
    expect = np.where(codes_lo % 2 == 0, pos[:-1], pos[1:])
    assert np.array_equal(got, expect)
    up = np.nextafter(mids32, np.float32(np.inf))
    dn = np.nextafter(mids32, np.float32(-np.inf))
    assert np.array_equal(E4M3_TORCH[oracle.e4m3_encode(up)], pos[1:])
    assert np.array_equal(E4M3_TORCH[oracle.e4m3_encode(dn)], pos[:-1])


def test_e4m3_encode_matches_library_cast_and_saturates():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(50),
        (rng.random(200000) * 463.9).astype(np.float32) * rng.choice([-1, 1], 200000).astype(np.float32),
        np.exp2(rng.uniform(-14, 8.85, 200000)).astype(np.float32),
    ])
    x = x[np.abs(x) < 464]
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = oracle.e4m3_encode(x)
    # +0 / -0 may differ only in sign for values that round to zero
    same = (lib == ours) | ((lib & 0x7F) == 0) & ((ours & 0x7F) == 0)
    assert same.all()
    big = np.array([448, 463.99, 464, 1e6, 3e38, np.inf], np.float32)
    assert (oracle.e4m3_encode(big) == 0x7E).all()
    assert (oracle.e4m3_encode(-big) == 0xFE).all()


def test_bf16_encode_matches_library_cast():
    rng = np.random.default_rng(2)
    bits = rng.integers(0, 2 ** 32, size=1 << 22, dtype=np.uint64).astype(np.uint32)
    # add every exponent with mantissa patterns next to the rounding boundary
    e = np.arange(256, dtype=np.uint32) << 23
    low = np.array([0x7FFF, 0x8000, 0x8001, 0x18000, 0x17FFF, 0x7FFFFF, 0], np.uint32)
    edge = (e[:, None] | low[None, :]).ravel()
    bits = np.concatenate([bits, edge, edge | 0x80000000])
    f = bits.view(np.float32)
    f = f[~np.isnan(f)]
    ours = oracle.bf16_encode(f)
    lib = bf16_bits(f)
    assert np.array_equal(ours, lib)
    assert np.array_equal(oracle.bf16_decode(ours), bf16_vals(lib))


# -------------------------------------------------------------- quantize ----
def _rand_bf16(shape, seed, scale=1.0, offset=None):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape).astype(np.float32) * np.float32(scale)
    if offset is not None:
        x = x + offset
    return bf16_bits(x)


def _qkv(B, Tq, Tkv, H, D, seed=0, koff=None):
    q = _rand_bf16((B, Tq, H, D), seed)
    k = _rand_bf16((B, Tkv, H, D), seed + 1, offset=koff)
    v = _rand_bf16((B, Tkv, H, D), seed + 2)
    return q, k, v


def test_quantize_half_step_bound_and_full_range():
    q, k, v = _qkv(2, 100, 150, 3, 128, seed=3, koff=np.float32(3.0))
    z = oracle.quantize(q, k, v)
    qf, kf, vf = bf16_vals(q), bf16_vals(k), bf16_vals(v)
    km = z["km"]
    for b in range(2):
        for h in range(3):
            for name, x, s8, scales, g, T in (("q", qf[b, :, h], z["q8"][b, h], z["sq"][b, h], 32, 100),
                                               ("k", kf[b, :, h] - km[b, h][None, :], z["k8"][b, h],
                                                z["sk"][b, h], 64, 150)):
                for gi, s in enumerate(scales):
                    rows = slice(gi * g, min(T, gi * g + g))
                    xs = x[rows].astype(np.float64)
                    w = s8[rows].astype(np.int64)
                    assert np.abs(w).max() == 127
                    # half a step, plus the rounding of inv = 127/amax and of x*inv (< 127 * 2^-21 steps)
                    assert np.all(np.abs(xs - w * np.float64(s)) <= np.float64(s) * (0.5 + 127 * 2.0 ** -21))
                    assert s == np.float32(np.abs(x[rows]).max()) / np.float32(127)


def test_quantize_power_of_two_invariance():
    q, k, v = _qkv(1, 64, 128, 2, 128, seed=5)
    z = oracle.quantize(q, k, v)
    for kexp in (-3, 5):
        f = np.float32(2.0 ** kexp)
        z2 = oracle.quantize(bf16_bits(bf16_vals(q) * f), bf16_bits(bf16_vals(k) * f), bf16_bits(bf16_vals(v) * f))
        for w in ("q8", "k8", "v8"):
            assert np.array_equal(z[w], z2[w])
        for s in ("sq", "sk", "sv", "km"):
            assert np.array_equal(z[s] * f, z2[s])


def test_k_smoothing_removes_channel_offset_exactly():
    # dyadic inputs: every sum, mean and difference below is exact, so adding a
    # per-channel constant to K must leave the K words and scales unchanged.
    rng = np.random.default_rng(7)
    B, T, H, D = 1, 128, 2, 128
    kx = (rng.integers(-64, 65, size=(B, T, H, D)) / 16.0).astype(np.float32)
    off = (rng.integers(-16, 17, size=(H, D)) / 4.0).astype(np.float32)
    q = bf16_bits(rng.standard_normal((B, T, H, D)))
    v = bf16_bits(rng.standard_normal((B, T, H, D)))
    z0 = oracle.quantize(q, bf16_bits(kx), v)
    z1 = oracle.quantize(q, bf16_bits(kx + off[None, None]), v)
    assert np.array_equal(z0["k8"], z1["k8"])
    assert np.array_equal(z0["sk"], z1["sk"])
    assert np.array_equal(z1["km"] - z0["km"], np.broadcast_to(off, (B, H, D)))


def test_k_mean_is_the_exact_mean_rounded():
    q, k, v = _qkv(1, 70, 197, 2, 128, seed=9, koff=np.float32(-1.5))
    z = oracle.quantize(q, k, v)
    kf = bf16_vals(k).astype(np.float64)
    for h in range(2):
        for d in range(0, 128, 7):
            exact = math.fsum(kf[0, :, h, d]) / 197
            assert z["km"][0, h, d] == np.float32(exact)


def test_v_fp8_half_step_bound():
    q, k, v = _qkv(1, 10, 300, 2, 128, seed=11)
    z = oracle.quantize(q, k, v)
    vf = bf16_vals(v).astype(np.float64)
    tab = E4M3_TORCH.astype(np.float64)
    for h in range(2):
        amax = np.abs(vf[0, :, h]).max(axis=0)
        assert np.array_equal(z["sv"][0, h], (amax.astype(np.float32) / np.float32(448)))
        y = vf[0, :, h] * (448.0 / amax)[None, :]
        dec = tab[z["v8"][0, h]]
        # E4M3: relative half-step 2^-4 for normals, absolute 2^-10 below 2^-6
        bound = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6)
        assert np.all(np.abs(dec - y) <= bound)


def test_quantize_ignores_tokens_beyond_T():
    q, k, v = _qkv(1, 96, 96, 1, 128, seed=13)
    junk = bf16_bits(np.full((1, 40, 1, 128), 1000.0))
    big = [np.concatenate([a, junk], axis=1) for a in (q, k, v)]
    z0 = oracle.quantize(q[:, :70], k[:, :70], v[:, :70])
    z1 = oracle.quantize(big[0][:, :70], big[1][:, :70], big[2][:, :70])
    for key in ("q8", "k8", "v8", "sq", "sk", "sv", "km"):
        assert np.array_equal(z0[key], z1[key])
    # the last partial groups use only their valid tokens
    assert z0["sq"].shape[-1] == 3 and z0["sk"].shape[-1] == 2


# ---------------------------------------------------------------- scores ----
def test_scores_equal_integer_matmul():
    q, k, v = _qkv(2, 130, 190, 2, 128, seed=15)
    z = oracle.quantize(q, k, v)
    for b, h in ((0, 1), (1, 0)):
        got = oracle.scores(z, b, h, 0, 130, 0, 190)
        ref = z["q8"][b, h].astype(np.int64) @ z["k8"][b, h].astype(np.int64).T
        assert np.array_equal(got, ref)


# --------------------------------------------------------------- softmax ----
def test_dequantized_scores_with_unit_scales():
    # A closed form of the score path: Q rows hold one channel of value 127 each, K keys
    # come in +127/-127 pairs per channel, so every K channel mean is exactly 0, every
    # scale is amax/127 = 1 and the words are the values themselves.  Then acc is in
    # {16129, -16129, 0} and t = float(acc) * ((sq*sk)*c) reduces to one rounding of
    # acc * c, with c = float(scale * log2(e)) taken in FP64 and rounded once.
    D, Tq, Tkv = 128, 5, 10
    qv = np.zeros((1, Tq, 1, D), np.float32)
    kv = np.zeros((1, Tkv, 1, D), np.float32)
    for i in range(Tq):
        qv[0, i, 0, (3 * i) % 5] = 127.0
    for j in range(Tkv):
        kv[0, j, 0, j // 2] = 127.0 if j % 2 == 0 else -127.0
    vv = np.ones((1, Tkv, 1, D), np.float32)
    z = oracle.quantize(bf16_bits(qv), bf16_bits(kv), bf16_bits(vv))
    assert np.all(z["km"] == 0) and np.all(z["sq"] == 1) and np.all(z["sk"] == 1)
    scale = 0.088388
    c = np.float32(np.float64(np.float32(scale)) * math.log2(math.e))
    assert oracle.log2_scale(scale) == c
    for i in range(Tq):
        tr = oracle.row_trace(z, scale, 64, 0, 0, i)
        acc = np.array([16129 * (1 if j % 2 == 0 else -1) if j // 2 == (3 * i) % 5 else 0 for j in range(Tkv)])
        assert np.array_equal(tr["acc"], acc)
        assert np.array_equal(tr["t"], (acc.astype(np.float32) * c).astype(np.float32))


@pytest.mark.parametrize("epoch", [64, 128])
def test_softmax_trace_invariants(epoch):
    q, k, v = _qkv(1, 40, 333, 1, 128, seed=17)
    z = oracle.quantize(q, k, v)
    c = oracle.log2_scale(1 / math.sqrt(128))
    for i in (0, 17, 39):
        tr = oracle.row_trace(z, 1 / math.sqrt(128), epoch, 0, 0, i)
        t = tr["t"].astype(np.float64)
        assert tr["m"][-1] == tr["t"].max()
        # rows sum to one: sum_j 2^(t_j - m) / d == 1
        assert abs(np.sum(np.exp2(t - tr["m"][-1])) / tr["d"][-1] - 1.0) < 1e-5
        # running max is the prefix max per epoch, alpha the ratio of successive maxima
        for e in range(len(tr["m"])):
            assert tr["m"][e] == tr["t"][: (e + 1) * epoch].max()
        assert tr["alpha"][0] == 0.0
        assert np.allclose(tr["alpha"][1:], np.exp2(tr["m"][:-1].astype(np.float64) - tr["m"][1:]), rtol=1e-6)
        # probability words: E4M3 of 448 * 2^(t - m_epoch) within half a step
        m_of_key = np.repeat(tr["m"], epoch)[: len(t)].astype(np.float64)
        y = 448.0 * np.exp2(t - m_of_key)
        dec = E4M3_TORCH[tr["p8"]].astype(np.float64)
        bound = np.maximum(y * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-5)
        assert np.all(np.abs(dec - y) <= bound)
        # the int32 scores are the exact dot products
        assert np.array_equal(tr["acc"], z["q8"][0, 0, i].astype(np.int64) @ z["k8"][0, 0].astype(np.int64).T)
        assert c == np.float32(1 / math.sqrt(128) * math.log2(math.e)) or abs(c / (1 / math.sqrt(128) / math.log(2)) - 1) < 1e-7


def test_epoch_size_changes_only_fp8_rounding():
    """d * 2^m (the normaliser) is independent of the epoch length up to FP32 rounding."""
    q, k, v = _qkv(1, 32, 500, 1, 128, seed=19)
    z = oracle.quantize(q, k, v)
    rows = np.array([[0, 0, i] for i in range(32)])
    res = {e: oracle.attend_rows(z, 0.0883883476, e, rows) for e in (64, 128, 500)}
    norm = {e: res[e][2].astype(np.float64) * np.exp2(res[e][1].astype(np.float64)) for e in res}
    assert np.allclose(norm[64], norm[500], rtol=2e-6)
    assert np.allclose(norm[128], norm[500], rtol=2e-6)
    o = {e: oracle.bf16_decode(res[e][0]).astype(np.float64) for e in res}
    rel = np.linalg.norm(o[64] - o[500]) / np.linalg.norm(o[500])
    assert rel < 3e-2


# ------------------------------------------------------- whole pipeline -----
def _fp64_attention(qf, kf, vf, scale):
    s = (qf @ kf.T) * scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p, p @ vf


@pytest.mark.parametrize("T", [4, 17, 64, 130])
def test_against_fp64_attention_with_derived_bound(T):
    D = 128
    q, k, v = _qkv(1, T, T, 1, D, seed=100 + T)
    z = oracle.quantize(q, k, v)
    scale = 1 / math.sqrt(D)
    out = oracle.bf16_decode(oracle.attend_all(z, scale, 64))[0, :, 0].astype(np.float64)
    qf, kf, vf = (bf16_vals(a)[0, :, 0].astype(np.float64) for a in (q, k, v))
    ks = kf - z["km"][0, 0][None, :].astype(np.float64)   # smoothing does not change softmax
    p, ref = _fp64_attention(qf, kf, vf, scale)
    # score perturbation from INT8 rounding: |q.k - q^.k^| <= (sk/2)*sum|q^| + (sq/2)*sum|k_s|
    sq = np.repeat(z["sq"][0, 0], 32)[:T].astype(np.float64)
    sk = np.repeat(z["sk"][0, 0], 64)[:T].astype(np.float64)
    qh = z["q8"][0, 0].astype(np.float64) * sq[:, None]
    dlt = scale * ((sk[None, :] / 2) * np.abs(qh).sum(1)[:, None] + (sq[:, None] / 2) * np.abs(ks).sum(1)[None, :])
    dmax = dlt.max(axis=1, keepdims=True)
    # FP8 P and FP8 V: relative 2^-4 each plus the subnormal floors; BF16 output 2^-8
    amax_v = np.abs(vf).max(axis=0)
    pv_abs = p @ np.abs(vf)
    bound = (pv_abs * (np.exp(2 * dmax) - 1 + 2 * 2.0 ** -4 + 2.0 ** -7)
             + (2.0 ** -10 / 448) * T * amax_v[None, :] * 2 + 2.0 ** -10 * amax_v[None, :] / 448 * 2
             + np.abs(ref) * 2.0 ** -8) * 1.05
    err = np.abs(out - ref)
    assert np.all(err <= bound), float((err / bound).max())
    rel = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert rel < 5e-2   # two E4M3 roundings of ~2.6% rms each set this level


def test_one_hot_permutation_v_closed_form():
    T, D = 100, 128
    rng = np.random.default_rng(23)
    perm = rng.permutation(D)[:T]
    vv = np.zeros((1, T, 1, D), np.float32)
    vv[0, np.arange(T), 0, perm] = 1.0
    q, k, _ = _qkv(1, T, T, 1, D, seed=29)
    z = oracle.quantize(q, k, bf16_bits(vv))
    scale = 1 / math.sqrt(D)
    out = oracle.bf16_decode(oracle.attend_all(z, scale, 64))[0, :, 0].astype(np.float64)
    unused = np.setdiff1d(np.arange(D), perm)
    assert np.all(out[:, unused] == 0)
    for i in (0, 50, 99):
        tr = oracle.row_trace(z, scale, 64, 0, 0, i)
        t = tr["t"].astype(np.float64)
        P = np.exp2(t - t.max())
        P /= P.sum()
        got = out[i, perm]
        assert np.all(np.abs(got - P) <= P * (2.0 ** -4 + 2.0 ** -7) + 2.0 ** -10 / 448 * 1.01 + 1e-12)


def test_v_power_of_two_scales_output_exactly():
    q, k, v = _qkv(1, 50, 200, 2, 128, seed=31)
    z = oracle.quantize(q, k, v)
    z2 = oracle.quantize(q, k, bf16_bits(bf16_vals(v) * np.float32(8)))
    o1 = oracle.bf16_decode(oracle.attend_all(z, 0.088, 64))
    o2 = oracle.bf16_decode(oracle.attend_all(z2, 0.088, 64))
    assert np.array_equal(o1 * np.float32(8), o2)


def test_brute_force_4x4_golden():
    g = json.load(open(os.path.join(GOLDEN, "brute4x4.json")))
    Q, K, V = (np.array(g[x], np.float32).reshape(1, 4, 1, 4) for x in ("Q", "K", "V"))
    z = oracle.quantize(bf16_bits(Q), bf16_bits(K), bf16_bits(V), gq=32, gk=64)
    assert np.array_equal(z["km"][0, 0], np.array(g["km"], np.float32))
    assert np.array_equal(z["q8"][0, 0], np.array(g["q8"]))
    assert np.array_equal(z["k8"][0, 0], np.array(g["k8"]))
    assert np.array_equal(z["v8"][0, 0], np.array(g["v8"]))
    assert np.array_equal(oracle.scores(z, 0, 0, 0, 4, 0, 4), np.array(g["acc"]))
    assert z["sq"][0, 0, 0] == np.float32(1) / np.float32(127)
    assert z["sk"][0, 0, 0] == np.float32(0.75) / np.float32(127)
    # direct (non-online) formula in FP64 on the hand-derived words: one max, one exp, one sum
    scale = 0.5
    acc = np.array(g["acc"], np.float64)
    f = float(np.float32(z["sq"][0, 0, 0]) * np.float32(z["sk"][0, 0, 0]) * np.float32(scale / math.log(2)))
    t = acc * f
    p = np.exp2(t - t.max(axis=1, keepdims=True))
    d = p.sum(axis=1, keepdims=True)
    p8 = E4M3_TORCH[torch.from_numpy((448 * p).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()]
    v8 = E4M3_TORCH[np.array(g["v8"])].astype(np.float64)
    amax = np.array(g["v_amax"], np.float64)
    expect = (p8 @ v8) / d * (amax / 448 / 448)[None, :]
    out = oracle.bf16_decode(oracle.attend_all(z, scale, 64))[0, :, 0].astype(np.float64)
    assert np.allclose(out, expect, rtol=2.0 ** -8, atol=0)

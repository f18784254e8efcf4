"""CPU oracle for SageAttention-style quantized self-attention (Python side).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline arm of ``bench.py`` may import this package; the product path
(``quantized_attention_video_b200``) never does.  The arithmetic lives in
``oracle.cpp`` (plain C++17, no fused multiply-add, OpenMP over independent
rows); this module only builds it and marshals numpy arrays.

Pins: every function here is checked against something other than itself by
the ``-m "not gpu"`` tests (format definitions and a library cast for the
codecs; invariants, closed forms, an FP64 unquantized attention and a
hand-derived 4x4 case for the policy).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_SO = os.path.join(_HERE, "liboracle.so")

GQ = 32   # Q tokens per INT8 scale group
GK = 64   # K tokens per INT8 scale group
EPOCH_PAGES = 64  # the pages' K64 epochs

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so next to it."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp"
        subprocess.check_call(["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                               "-shared", "-fPIC", "-o", tmp, _SRC])
        os.replace(tmp, _SO)
    return _SO


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.orc_bf16_decode.restype = _F
        L.orc_bf16_decode.argtypes = [ctypes.c_uint16]
        L.orc_bf16_encode.restype = ctypes.c_uint16
        L.orc_bf16_encode.argtypes = [_F]
        L.orc_e4m3_decode.restype = _F
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [_F]
        L.orc_bf16_encode_array.argtypes = [_P, _P, _I64]
        L.orc_e4m3_encode_array.argtypes = [_P, _P, _I64]
        L.orc_log2_scale.restype = _F
        L.orc_log2_scale.argtypes = [_F]
        L.orc_quantize.argtypes = [_P, _P, _P] + [_I64] * 9 + [_I] * 7 + [_P] * 7
        L.orc_scores.argtypes = [_P, _P] + [_I] * 5 + [_I] * 6 + [_P]
        L.orc_attend_rows.argtypes = [_P] * 6 + [_I] * 7 + [_F, _I, _I, _P, _P, _P, _P]
        L.orc_row_trace.argtypes = [_P] * 6 + [_I] * 7 + [_F, _I, _I, _I, _I] + [_P] * 9
        L.orc_qk_norm_rope.argtypes = [_P, _I64, _I64, _I64, _I, _I, _I, _I, _P, _F, _P, _P, _P]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


# ------------------------------------------------------------------ codecs --
def bf16_encode(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().orc_bf16_encode_array(x.ctypes.data, out.ctypes.data, x.size)
    return out


def bf16_decode(h) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


def e4m3_encode(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_array(x.ctypes.data, out.ctypes.data, x.size)
    return out


def e4m3_decode_table() -> np.ndarray:
    return np.array([lib().orc_e4m3_decode(i) for i in range(256)], dtype=np.float32)


def log2_scale(scale: float) -> float:
    return lib().orc_log2_scale(scale)


# ---------------------------------------------------------------- quantize --
def _view_args(a):
    """Base pointer and element strides (b, t, h) of a [B,T,H,D] uint16 view with unit d stride."""
    assert a.dtype == np.uint16 and a.ndim == 4
    assert a.strides[3] == 2, "channel stride must be one element"
    sb, st, sh = (s // 2 for s in a.strides[:3])
    return a.ctypes.data, sb, st, sh


def quantize(q, k, v, gq: int = GQ, gk: int = GK) -> dict:
    """Quantize BF16 Q/K/V views ([B,T,H,D] uint16, any strides with unit d stride)."""
    B, Tq, H, D = q.shape
    Tkv = k.shape[1]
    assert k.shape == (B, Tkv, H, D) and v.shape == (B, Tkv, H, D)
    nq, nk = -(-Tq // gq), -(-Tkv // gk)
    r = dict(
        km=np.empty((B, H, D), np.float32), sq=np.empty((B, H, nq), np.float32),
        sk=np.empty((B, H, nk), np.float32), sv=np.empty((B, H, D), np.float32),
        q8=np.empty((B, H, Tq, D), np.int8), k8=np.empty((B, H, Tkv, D), np.int8),
        v8=np.empty((B, H, Tkv, D), np.uint8),
    )
    qa, ka, va = _view_args(q), _view_args(k), _view_args(v)
    rc = lib().orc_quantize(qa[0], ka[0], va[0], *qa[1:], *ka[1:], *va[1:], B, Tq, Tkv, H, D, gq, gk,
                            *(r[x].ctypes.data for x in ("km", "sq", "sk", "sv", "q8", "k8", "v8")))
    if rc != 0:
        raise ValueError("orc_quantize rejected its arguments")
    r.update(B=B, Tq=Tq, Tkv=Tkv, H=H, D=D, gq=gq, gk=gk)
    return r


def qk_norm_rope(x, gamma, eps: float, cos, sin) -> np.ndarray:
    """Per-head RMSNorm + interleaved-pair RoPE of a BF16 [B,T,H,D] view (oracle.cpp,
    orc_qk_norm_rope, for the exact steps).  gamma [D], cos/sin [T, D/2] FP32.
    Returns a dense [B,T,H,D] uint16 (BF16 bits) array."""
    B, T, H, D = x.shape
    gamma = np.ascontiguousarray(gamma, dtype=np.float32)
    cos = np.ascontiguousarray(cos, dtype=np.float32)
    sin = np.ascontiguousarray(sin, dtype=np.float32)
    assert gamma.shape == (D,) and cos.shape == (T, D // 2) and sin.shape == (T, D // 2)
    out = np.empty((B, T, H, D), np.uint16)
    xa = _view_args(x)
    rc = lib().orc_qk_norm_rope(xa[0], *xa[1:], B, T, H, D, gamma.ctypes.data, eps, cos.ctypes.data,
                                sin.ctypes.data, out.ctypes.data)
    if rc != 0:
        raise ValueError("orc_qk_norm_rope rejected its arguments")
    return out


def quantize_norm_rope(q, k, v, nr: dict, gq: int = GQ, gk: int = GK) -> dict:
    """The preparation with Q/K RMSNorm + RoPE: qk_norm_rope on Q and on K, then quantize.
    nr holds gamma_q, gamma_k, eps, cos_q, sin_q, cos_k, sin_k."""
    qn = qk_norm_rope(q, nr["gamma_q"], nr["eps"], nr["cos_q"], nr["sin_q"])
    kn = qk_norm_rope(k, nr["gamma_k"], nr["eps"], nr["cos_k"], nr["sin_k"])
    return quantize(qn, kn, v, gq, gk)


def _qz_args(z):
    return (z["q8"].ctypes.data, z["k8"].ctypes.data, z["v8"].ctypes.data, z["sq"].ctypes.data,
            z["sk"].ctypes.data, z["sv"].ctypes.data, z["B"], z["Tq"], z["Tkv"], z["H"], z["D"],
            z["gq"], z["gk"])


def scores(z, b, h, i0, ni, j0, nj) -> np.ndarray:
    out = np.empty((ni, nj), np.int32)
    rc = lib().orc_scores(z["q8"].ctypes.data, z["k8"].ctypes.data, z["B"], z["Tq"], z["Tkv"], z["H"], z["D"],
                          b, h, i0, ni, j0, nj, out.ctypes.data)
    if rc != 0:
        raise ValueError("orc_scores rejected its arguments")
    return out


def attend_rows(z, scale: float, epoch: int, rows) -> tuple:
    """Rows = int array [n, 3] of (b, h, i).  Returns (out uint16 [n, D], m [n], d [n])."""
    rows = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
    n = rows.shape[0]
    out = np.empty((n, z["D"]), np.uint16)
    m = np.empty(n, np.float32)
    d = np.empty(n, np.float32)
    rc = lib().orc_attend_rows(*_qz_args(z), scale, epoch, n, rows.ctypes.data, out.ctypes.data,
                               m.ctypes.data, d.ctypes.data)
    if rc != 0:
        raise ValueError("orc_attend_rows rejected its arguments")
    return out, m, d


def attend_all(z, scale: float, epoch: int) -> np.ndarray:
    """All outputs as a [B, Tq, H, D] uint16 (BF16 bits) array."""
    B, Tq, H = z["B"], z["Tq"], z["H"]
    bb, hh, ii = np.meshgrid(np.arange(B), np.arange(H), np.arange(Tq), indexing="ij")
    rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], axis=1)
    out, _, _ = attend_rows(z, scale, epoch, rows)
    return out.reshape(B, H, Tq, z["D"]).transpose(0, 2, 1, 3).copy()


def row_trace(z, scale: float, epoch: int, b: int, h: int, i: int) -> dict:
    Tkv, D = z["Tkv"], z["D"]
    ne = -(-Tkv // epoch)
    tr = dict(out=np.empty(D, np.uint16), acc=np.empty(Tkv, np.int32), t=np.empty(Tkv, np.float32),
              p8=np.empty(Tkv, np.uint8), m=np.empty(ne, np.float32), d=np.empty(ne, np.float32),
              alpha=np.empty(ne, np.float32), ro=np.empty(D, np.float32), r=np.empty(1, np.float32))
    rc = lib().orc_row_trace(*_qz_args(z), scale, epoch, b, h, i,
                             *(tr[x].ctypes.data for x in ("out", "acc", "t", "p8", "m", "d", "alpha", "ro", "r")))
    if rc != 0:
        raise ValueError("orc_row_trace rejected its arguments")
    return tr

"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

Holds none of the attention method's arithmetic: only the workload shapes and
the recipes that draw BF16 Q/K/V (``gen.c``).  The five workloads mirror the
shapes of the H3 video-diffusion attention described on the pages:

* ``fixed_q128_kv192``: the fixed single-tile shape of the aligned numerical
  prototype ("Phase 2B Aligned Numerical Prototype", Decision): B=1, H=1,
  Tq=128, Tkv=192, D=128, N(0,1) values.
* ``selfattn_h8_t4096``: B=1, H=8, T=4096; K has a per-channel offset drawn
  from N(0, 4) (std 2) to exercise K mean-smoothing.
* ``ragged_h16_t9453``: B=1, H=16, T=9453 (not a multiple of 64 or 128); Q/K
  RMS-normalised per (token, head) and scaled by gamma ~ N(1, 0.1).
* ``h3_t37810_h32``: the H3 packed video+text sequence of the representative
  workload ("H3 Performance Roadmap", Measured GB10 Baseline: 37,810 packed
  tokens), H=32, D=128, Q/K RMS-normed with gamma.
* ``h3_packed_b2_t37810``: the same shape with batch 2 read from one packed
  [2, T, 3, H, D] QKV buffer, output into [2, T, H*D].

N(mu, v) names a normal with variance v.

Workloads with ``norm_rope`` set feed raw projection-like Q/K (N(0,1)) through the
Q/K RMSNorm + RoPE preparation: per-channel weights gamma_q, gamma_k ~ N(1, 0.1),
eps = 1e-6, and rotary tables from ``rope_tables``: video tokens laid out in
raster order on frames of 24 x 42 latent tokens, the 64 channel pairs split
8 / 28 / 28 between the time, height and width positions, pair k of an axis with
n pairs turning at theta^(-k/n) radians per position (theta = 256); the last 100
tokens (the text) are left unrotated (cos 1, sin 0).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_SRC = os.path.join(_HERE, "gen.c")

NORMAL, OFFSET, RMSNORM = 0, 1, 2
STREAM_Q, STREAM_K, STREAM_V, STREAM_GAMMA_Q, STREAM_GAMMA_K, STREAM_OFFSET_K, STREAM_NR_GAMMA_Q, STREAM_NR_GAMMA_K = \
    range(8)
ROPE_THETA = 256.0
ROPE_PAIRS = (8, 28, 28)  # time, height, width (64 channel pairs)
ROPE_FRAME = (24, 42)     # latent tokens per frame: height x width, raster order
ROPE_TEXT = 100           # trailing tokens left unrotated
NORM_EPS = 1e-6


def build(force: bool = False) -> str:
    """Compile gen.c into libsynth.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.synth_normal_f32.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                         ctypes.c_uint32, ctypes.c_double, ctypes.c_double]
        lib.synth_fill_bf16.argtypes = [ctypes.c_void_p] + [ctypes.c_int] * 4 + [ctypes.c_int64] * 3 + [
            ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_void_p]
        _lib = lib
    return _lib


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Tq: int
    Tkv: int
    H: int
    D: int
    recipe: str          # "normal", "k_offset" or "rmsnorm"
    seed: int
    packed: bool = False  # Q/K/V read from one [B,T,3,H,D] buffer, out [B,T,H*D]
    norm_rope: bool = False  # Q/K pass through the RMSNorm + RoPE preparation

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))

    @property
    def ops(self) -> float:
        """Algorithmic tensor operations of one call: 2*D per score for QK and 2*D for PV."""
        return 4.0 * self.B * self.Tq * self.Tkv * self.H * self.D


WORKLOADS = {
    "fixed_q128_kv192": Workload("fixed_q128_kv192", 1, 128, 192, 1, 128, "normal", 73021),
    "selfattn_h8_t4096": Workload("selfattn_h8_t4096", 1, 4096, 4096, 8, 128, "k_offset", 4096),
    "ragged_h16_t9453": Workload("ragged_h16_t9453", 1, 9453, 9453, 16, 128, "rmsnorm", 9453),
    "h3_t37810_h32": Workload("h3_t37810_h32", 1, 37810, 37810, 32, 128, "rmsnorm", 37810),
    "h3_packed_b2_t37810": Workload("h3_packed_b2_t37810", 2, 37810, 37810, 32, 128, "rmsnorm", 37811,
                                    packed=True),
    # the pages' second required shape, "74K tokens" (the 243-frame workload), read as 74,000
    "h3_t74000_h32": Workload("h3_t74000_h32", 1, 74000, 74000, 32, 128, "rmsnorm", 74000),
    # raw Q/K through the Q/K RMSNorm + RoPE preparation
    "nr_h4_t1100": Workload("nr_h4_t1100", 1, 1100, 1100, 4, 128, "normal", 1100, norm_rope=True),
    "h3_t37810_h32_nr": Workload("h3_t37810_h32_nr", 1, 37810, 37810, 32, 128, "normal", 37812,
                                 norm_rope=True),
}


def rope_tables(T: int, n_text: int = ROPE_TEXT, frame=ROPE_FRAME, pairs=ROPE_PAIRS, theta: float = ROPE_THETA):
    """Rotary tables cos, sin [T, 64] float32 of the layout described in the module docstring."""
    assert sum(pairs) == 64
    n_vid = max(0, T - n_text)
    v = np.arange(n_vid)
    per_frame = frame[0] * frame[1]
    pos = (v // per_frame, (v % per_frame) // frame[1], v % frame[1])
    ang = np.zeros((T, 64), dtype=np.float64)
    col = 0
    for axis, n in enumerate(pairs):
        freq = theta ** (-np.arange(n, dtype=np.float64) / n)
        ang[:n_vid, col:col + n] = pos[axis][:, None].astype(np.float64) * freq[None, :]
        col += n
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def norm_rope_params(w: "Workload") -> dict:
    """Host (numpy) parameters of the Q/K RMSNorm + RoPE of a norm_rope workload."""
    cq, sq = rope_tables(w.Tq)
    ck, sk = (cq, sq) if w.Tkv == w.Tq else rope_tables(w.Tkv)
    return dict(gamma_q=normal_f32(w.D, w.seed, STREAM_NR_GAMMA_Q, 1.0, float(np.sqrt(0.1))),
                gamma_k=normal_f32(w.D, w.seed, STREAM_NR_GAMMA_K, 1.0, float(np.sqrt(0.1))),
                eps=NORM_EPS, cos_q=cq, sin_q=sq, cos_k=ck, sin_k=sk)


def normal_f32(n: int, seed: int, stream: int, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _load().synth_normal_f32(out.ctypes.data, n, seed, stream, mean, std)
    return out


def fill_bf16(out: np.ndarray, B: int, T: int, H: int, D: int, strides, seed: int, stream: int,
              kind: int = NORMAL, mean: float = 0.0, std: float = 1.0, vec: np.ndarray | None = None,
              offset_elems: int = 0):
    """Fill the logical [B,T,H,D] view at ``out.flat[offset_elems:]`` with element strides (sb, st, sh).

    ``out`` is a C-contiguous uint16 array (BF16 bit patterns) that must span the whole view.
    """
    assert out.dtype == np.uint16 and out.flags.c_contiguous
    assert D <= 1024
    sb, st, sh = strides
    last = offset_elems + (B - 1) * sb + (T - 1) * st + (H - 1) * sh + D
    assert 0 <= offset_elems and last <= out.size
    if kind != NORMAL:
        assert vec is not None and vec.dtype == np.float32 and vec.size == H * D
        vec = np.ascontiguousarray(vec)
    _load().synth_fill_bf16(out.ctypes.data + 2 * offset_elems, B, T, H, D, sb, st, sh, seed, stream,
                            kind, mean, std, None if vec is None else vec.ctypes.data)


def _fill_tensor(out, w: Workload, T: int, strides, which: str, offset_elems: int = 0):
    stream = {"q": STREAM_Q, "k": STREAM_K, "v": STREAM_V}[which]
    H, D = w.H, w.D
    kw = dict(offset_elems=offset_elems)
    if which == "v" or w.recipe == "normal" or (w.recipe == "k_offset" and which == "q"):
        fill_bf16(out, w.B, T, H, D, strides, w.seed, stream, **kw)
    elif w.recipe == "k_offset":
        off = normal_f32(H * D, w.seed, STREAM_OFFSET_K, 0.0, 2.0)
        fill_bf16(out, w.B, T, H, D, strides, w.seed, stream, OFFSET, vec=off, **kw)
    elif w.recipe == "rmsnorm":
        gstream = STREAM_GAMMA_Q if which == "q" else STREAM_GAMMA_K
        gamma = normal_f32(H * D, w.seed, gstream, 1.0, float(np.sqrt(0.1)))
        fill_bf16(out, w.B, T, H, D, strides, w.seed, stream, RMSNORM, vec=gamma, **kw)
    else:
        raise ValueError(w.recipe)


def make_separate(w: Workload):
    """Q [B,Tq,H,D], K and V [B,Tkv,H,D], contiguous uint16 BF16 bit patterns."""
    out = {}
    for which, T in (("q", w.Tq), ("k", w.Tkv), ("v", w.Tkv)):
        a = np.empty((w.B, T, w.H, w.D), dtype=np.uint16)
        _fill_tensor(a, w, T, (T * w.H * w.D, w.H * w.D, w.D), which)
        out[which] = a
    return out


def make_packed(w: Workload):
    """One packed [B,T,3,H,D] uint16 buffer (Tq == Tkv); slot 0 = Q, 1 = K, 2 = V."""
    assert w.Tq == w.Tkv
    T, H, D = w.Tq, w.H, w.D
    buf = np.empty((w.B, T, 3, H, D), dtype=np.uint16)
    strides = (T * 3 * H * D, 3 * H * D, D)
    for slot, which in enumerate(("q", "k", "v")):
        _fill_tensor(buf, w, T, strides, which, offset_elems=slot * H * D)
    return buf


def make_inputs(w: Workload):
    """Inputs for a workload: dict with 'q','k','v' logical [B,T,H,D] views (and 'packed' if packed)."""
    if w.packed:
        buf = make_packed(w)
        return {"packed": buf, "q": buf[:, :, 0], "k": buf[:, :, 1], "v": buf[:, :, 2]}
    return make_separate(w)

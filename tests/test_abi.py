"""C-ABI library checks that need no GPU: it loads, exports every symbol the
header declares, sizes its workspace, and rejects bad arguments before any
CUDA call (so nothing here touches a device)."""
import ctypes
import os
import re

import pytest

import quantized_attention_video_b200 as h3

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "h3attn.h")


@pytest.fixture(scope="module")
def L():
    from quantized_attention_video_b200 import build
    build.build()
    return h3.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(h3attn_\w+)\s*\(", text)))


def test_exports_every_declared_function(L):
    names = declared_functions()
    assert len(names) >= 10
    raw = ctypes.CDLL(h3.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    assert h3.h3attn_version() == 1


def test_status_strings(L):
    for s in range(7):
        assert h3.h3attn_status_string(s)
    assert h3.h3attn_status_string(99) == "unknown status"


def test_workspace_layout_matches_field_sizes(L):
    B, Tq, Tkv, H = 2, 300, 9453, 3
    off = h3.h3attn_workspace_layout(B, Tq, Tkv, H)
    Tqp, Tkp = 384, 9472
    nchunk = -(-Tkv // 64)
    # the INT8 Q/K words are held as BF16 values (2 bytes each)
    need = {"status": 256, "q8": 2 * B * H * Tqp * 128, "k8": 2 * B * H * Tkp * 128, "v8t": B * H * 128 * Tkp,
            "sq": B * H * Tqp // 32 * 4, "sk": B * H * Tkp // 64 * 4, "km": B * H * 128 * 4,
            "sv": B * H * 128 * 4, "ksum": B * H * nchunk * 128 * 8, "vmax": B * H * nchunk * 128 * 4}
    names = h3.WS_FIELDS
    for a, b in zip(names[:-1], names[1:]):
        assert off[a] % 1024 == 0
        assert off[b] - off[a] >= need[a]
        assert off[b] - off[a] < need[a] + 1024
    assert h3.h3attn_workspace_bytes(B, Tq, Tkv, H) == off["end"]


@pytest.mark.parametrize("args", [(0, 10, 10, 1, 128), (1, 0, 10, 1, 128), (1, 10, 0, 1, 128), (1, 10, 10, 0, 128),
                                  (1, 10, 10, 1, 64), (1, 10, 10, 70000, 128)])
def test_workspace_bytes_rejects_bad_sizes(L, args):
    assert h3.h3attn_workspace_bytes(*args) == 0


def _view(ptr, sb=3 * 4096, st=4096, sh=128):
    return h3._View(ptr, sb, st, sh)


def _forward(L, q, k, v, B=1, T=256, H=32, D=128, scale=0.088, out=None, ws=0x1000000, wsb=1 << 40):
    out = out if out is not None else _view(0x2000000)
    return L.h3attn_forward(ctypes.byref(q) if q is not None else None, ctypes.byref(k), ctypes.byref(v), B, T, H, D,
                            scale, ctypes.byref(out), ws, wsb, None)


def test_argument_errors_are_reported_without_a_device(L):
    good = _view(0x100000)
    assert _forward(L, None, good, good) == h3.ERR_INVALID_ARG
    assert _forward(L, good, good, good, D=64) == h3.ERR_UNSUPPORTED
    assert _forward(L, good, good, good, T=0) == h3.ERR_INVALID_ARG
    assert _forward(L, _view(0x100008), good, good) == h3.ERR_ALIGNMENT
    assert _forward(L, _view(0x100000, st=4100), good, good) == h3.ERR_ALIGNMENT
    assert _forward(L, _view(0), good, good) == h3.ERR_INVALID_ARG
    assert _forward(L, good, good, good, scale=0.0) == h3.ERR_INVALID_ARG
    assert _forward(L, good, good, good, scale=float("nan")) == h3.ERR_INVALID_ARG
    assert _forward(L, good, good, good, out=_view(0x2000004)) == h3.ERR_ALIGNMENT
    assert _forward(L, good, good, good, ws=0) == h3.ERR_WORKSPACE
    assert _forward(L, good, good, good, ws=0x1000080) == h3.ERR_WORKSPACE
    assert _forward(L, good, good, good, wsb=1000) == h3.ERR_WORKSPACE


def test_debug_export_rejects_out_of_range_tiles(L):
    ws = 0x1000000
    f = L.h3attn_debug_qk_scores
    assert f(ws, 1 << 40, 1, 256, 256, 2, 128, 0, 0, 2, 0, 0x3000000, None) == h3.ERR_INVALID_ARG
    assert f(ws, 1 << 40, 1, 256, 256, 2, 128, 0, 2, 0, 0, 0x3000000, None) == h3.ERR_INVALID_ARG
    assert f(ws, 1 << 40, 1, 256, 256, 2, 128, 0, 0, 0, 0, 0, None) == h3.ERR_INVALID_ARG
    assert f(ws, 1 << 40, 1, 256, 256, 2, 128, 0, 0, 0, 0, 0x3000004, None) == h3.ERR_ALIGNMENT


def test_host_pipeline_sizes_and_argument_errors(L):
    assert h3.h3attn_forward_host_bytes(1, 300, 300, 4, 0) == 0
    assert h3.h3attn_forward_host_bytes(1, 300, 300, 4, 5) == 0
    assert h3.h3attn_forward_host_bytes(1, 300, 300, 4, 2) == 2 * (h3.h3attn_forward_host_bytes(1, 300, 300, 2, 2) // 2)
    good = _view(0x100000)
    f = L.h3attn_forward_host
    args = lambda q=good, out=None, g=2, buf=0x4000000, nbytes=1 << 40, D=128: f(
        ctypes.byref(q) if q is not None else None, ctypes.byref(good), ctypes.byref(good), 1, 256, 256, 4, D, 0.088,
        ctypes.byref(out if out is not None else _view(0x2000000)), g, buf, nbytes, None)
    assert args(q=None) == h3.ERR_INVALID_ARG
    assert args(g=0) == h3.ERR_INVALID_ARG
    assert args(D=64) == h3.ERR_UNSUPPORTED
    assert args(q=_view(0x100008)) == h3.ERR_ALIGNMENT
    assert args(out=_view(0x2000000, st=4100)) == h3.ERR_ALIGNMENT
    assert args(buf=0) == h3.ERR_WORKSPACE
    assert args(buf=0x4000100) == h3.ERR_WORKSPACE
    assert args(nbytes=1000) == h3.ERR_WORKSPACE


def test_norm_rope_argument_errors(L):
    good = _view(0x100000)
    tab = 0x5000000

    def nr(**kw):
        f = dict(gamma_q=tab, gamma_k=tab, cos_q=tab, sin_q=tab, cos_k=tab, sin_k=tab, eps=1e-6)
        f.update(kw)
        return h3._NormRope(*(f[n] for n in h3.NORM_ROPE_FIELDS), f["eps"])

    def fwd(n, D=128):
        return L.h3attn_forward_norm_rope(ctypes.byref(good), ctypes.byref(good), ctypes.byref(good), 1, 256, 256, 4,
                                          D, 0.088, ctypes.byref(n) if n is not None else None,
                                          ctypes.byref(_view(0x2000000)), 0x1000000, 1 << 40, None)

    assert fwd(None) == h3.ERR_INVALID_ARG
    assert fwd(nr(), D=64) == h3.ERR_UNSUPPORTED
    assert fwd(nr(cos_k=0)) == h3.ERR_INVALID_ARG
    assert fwd(nr(gamma_q=tab + 4)) == h3.ERR_ALIGNMENT
    assert fwd(nr(eps=0.0)) == h3.ERR_INVALID_ARG
    assert fwd(nr(eps=float("inf"))) == h3.ERR_INVALID_ARG
    q = L.h3attn_quantize_qkv_norm_rope
    assert q(ctypes.byref(good), ctypes.byref(good), ctypes.byref(good), 1, 256, 256, 4, 128, None, 0x1000000,
             1 << 40, None) == h3.ERR_INVALID_ARG
    assert q(ctypes.byref(good), ctypes.byref(good), ctypes.byref(good), 1, 256, 256, 4, 128, ctypes.byref(nr()), 0,
             1 << 40, None) == h3.ERR_WORKSPACE
    f = L.h3attn_norm_rope
    out = _view(0x2000000)
    assert f(ctypes.byref(good), 1, 256, 4, 128, tab, tab, 0, 1e-6, ctypes.byref(out), None) == h3.ERR_INVALID_ARG
    assert f(ctypes.byref(good), 1, 256, 4, 128, tab, tab + 8, tab, 1e-6, ctypes.byref(out), None) == h3.ERR_ALIGNMENT
    assert f(ctypes.byref(good), 1, 256, 4, 128, tab, tab, tab, -1.0, ctypes.byref(out), None) == h3.ERR_INVALID_ARG
    assert f(ctypes.byref(_view(0x100004)), 1, 256, 4, 128, tab, tab, tab, 1e-6, ctypes.byref(out),
             None) == h3.ERR_ALIGNMENT
    assert f(ctypes.byref(good), 1, 0, 4, 128, tab, tab, tab, 1e-6, ctypes.byref(out), None) == h3.ERR_INVALID_ARG


def test_product_path_has_no_oracle_or_cpu_fallback():
    pkg = os.path.join(ROOT, "quantized_attention_video_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "liboracle" not in text, fn


def test_host_pipeline_group_layout(L):
    """Groups of heads_per_group heads, the first and the last halved once there are more
    than two full groups' worth of heads."""
    assert h3.h3attn_forward_host_groups(32, 2) == [0] + list(range(1, 32, 2)) + [31, 32][1:]
    assert h3.h3attn_forward_host_groups(8, 2) == [0, 1, 3, 5, 7, 8]
    assert h3.h3attn_forward_host_groups(10, 3) == [0, 1, 4, 7, 9, 10]
    assert h3.h3attn_forward_host_groups(4, 2) == [0, 2, 4]      # no room for halved ends
    assert h3.h3attn_forward_host_groups(5, 1) == [0, 1, 2, 3, 4, 5]
    assert h3.h3attn_forward_host_groups(7, 7) == [0, 7]
    for H in range(1, 40):
        for g in range(1, H + 1):
            s = h3.h3attn_forward_host_groups(H, g)
            sizes = [b - a for a, b in zip(s, s[1:])]
            assert s[0] == 0 and s[-1] == H and all(1 <= n <= g for n in sizes), (H, g, s)
    assert L.h3attn_forward_host_groups(8, 0, None) == 0
    assert L.h3attn_forward_host_groups(8, 9, None) == 0

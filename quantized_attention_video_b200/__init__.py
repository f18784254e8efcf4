"""Python binding of libh3attn.so (quantized dense self-attention for B200).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of the shared library, reached through its C ABI with ctypes.  The
functions carry the C names (``h3attn_forward`` ...) and take PyTorch CUDA
tensors for device memory; PyTorch is used for nothing else.

If the library has not been built this module raises on first use; there is
no CPU fallback.  Build it with ``python -m quantized_attention_video_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libh3attn.so")

HEAD_DIM = 128
TILE = 128
Q_GROUP = 32
K_GROUP = 64

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(7)
WS_FIELDS = ("status", "q8", "k8", "v8t", "sq", "sk", "km", "sv", "ksum", "vmax", "end")


class H3AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {h3attn_status_string(status)} (status {status})")
        self.status = status


class _View(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("stride_b", ctypes.c_int64), ("stride_t", ctypes.c_int64),
                ("stride_h", ctypes.c_int64)]


class _NormRope(ctypes.Structure):
    _fields_ = [("gamma_q", ctypes.c_void_p), ("gamma_k", ctypes.c_void_p), ("cos_q", ctypes.c_void_p),
                ("sin_q", ctypes.c_void_p), ("cos_k", ctypes.c_void_p), ("sin_k", ctypes.c_void_p),
                ("eps", ctypes.c_float)]


NORM_ROPE_FIELDS = ("gamma_q", "gamma_k", "cos_q", "sin_q", "cos_k", "sin_k")

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libh3attn.so; raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m quantized_attention_video_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        I, P, S, F, I64 = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float, ctypes.c_int64
        VP = ctypes.POINTER(_View)
        L.h3attn_workspace_bytes.restype = S
        L.h3attn_workspace_bytes.argtypes = [I] * 5
        L.h3attn_workspace_layout.restype = I
        L.h3attn_workspace_layout.argtypes = [I] * 5 + [ctypes.POINTER(I64)]
        L.h3attn_quantize_qkv.restype = I
        L.h3attn_quantize_qkv.argtypes = [VP, VP, VP] + [I] * 5 + [P, S, P]
        L.h3attn_attend.restype = I
        L.h3attn_attend.argtypes = [P, S] + [I] * 5 + [F, VP, P]
        L.h3attn_forward.restype = I
        L.h3attn_forward.argtypes = [VP, VP, VP] + [I] * 4 + [F, VP, P, S, P]
        L.h3attn_forward_ex.restype = I
        L.h3attn_forward_ex.argtypes = [VP, VP, VP] + [I] * 5 + [F, VP, P, S, P]
        L.h3attn_forward_static.restype = I
        L.h3attn_forward_static.argtypes = [VP, VP, VP] + [I] * 5 + [F, VP, P]
        L.h3attn_static_workspace_bytes.restype = S
        L.h3attn_static_workspace_bytes.argtypes = []
        L.h3attn_static_check_status.restype = I
        L.h3attn_static_check_status.argtypes = [P]
        L.h3attn_debug_static_attend_timeout.restype = I
        L.h3attn_debug_static_attend_timeout.argtypes = [I] * 5 + [F, VP, ctypes.c_uint64, P]
        L.h3attn_check_status.restype = I
        L.h3attn_check_status.argtypes = [P, P]
        L.h3attn_debug_qk_scores.restype = I
        L.h3attn_debug_qk_scores.argtypes = [P, S] + [I] * 9 + [P, P]
        L.h3attn_debug_attend_trace.restype = I
        L.h3attn_debug_attend_trace.argtypes = [P, S] + [I] * 5 + [F, VP, I, P, P]
        L.h3attn_debug_attend_timeout.restype = I
        L.h3attn_debug_attend_timeout.argtypes = [P, S] + [I] * 5 + [F, VP, ctypes.c_uint64, P]
        L.h3attn_forward_host_bytes.restype = S
        L.h3attn_forward_host_bytes.argtypes = [I] * 6
        L.h3attn_forward_host_groups.restype = I
        L.h3attn_forward_host_groups.argtypes = [I, I, P]
        L.h3attn_forward_host.restype = I
        L.h3attn_forward_host.argtypes = [VP, VP, VP] + [I] * 5 + [F, VP, I, P, S, P]
        L.h3attn_forward_host_check_status.restype = I
        L.h3attn_forward_host_check_status.argtypes = [P] + [I] * 6 + [P]
        L.h3attn_debug_forward_host_timeout.restype = I
        L.h3attn_debug_forward_host_timeout.argtypes = [VP, VP, VP] + [I] * 5 + [F, VP, I, P, S, I,
                                                                                  ctypes.c_uint64, P]
        NP = ctypes.POINTER(_NormRope)
        L.h3attn_quantize_qkv_norm_rope.restype = I
        L.h3attn_quantize_qkv_norm_rope.argtypes = [VP, VP, VP] + [I] * 5 + [NP, P, S, P]
        L.h3attn_forward_norm_rope.restype = I
        L.h3attn_forward_norm_rope.argtypes = [VP, VP, VP] + [I] * 5 + [F, NP, VP, P, S, P]
        L.h3attn_norm_rope.restype = I
        L.h3attn_norm_rope.argtypes = [VP] + [I] * 4 + [P, P, P, F, VP, P]
        L.h3attn_status_string.restype = ctypes.c_char_p
        L.h3attn_status_string.argtypes = [I]
        L.h3attn_version.restype = I
        L.h3attn_version.argtypes = []
        _lib = L
    return _lib


# ------------------------------------------------------------- marshalling --
def _view(t) -> _View:
    """[B, T, H, D] BF16 tensor (any strides, unit channel stride) -> view struct."""
    if t.dim() != 4:
        raise ValueError("expected a [B, T, H, D] tensor")
    if t.stride(3) != 1:
        raise ValueError("channel stride must be 1")
    return _View(t.data_ptr(), t.stride(0), t.stride(1), t.stride(2))


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _ptr_bytes(ws):
    return ws.data_ptr(), ws.numel() * ws.element_size()


def _check(st: int, where: str):
    if st != OK:
        raise H3AttnError(st, where)


# -------------------------------------------------------------- C names ----
def h3attn_status_string(status: int) -> str:
    return lib().h3attn_status_string(status).decode()


def h3attn_version() -> int:
    return lib().h3attn_version()


def h3attn_workspace_bytes(B: int, Tq: int, Tkv: int, H: int, D: int = HEAD_DIM) -> int:
    return lib().h3attn_workspace_bytes(B, Tq, Tkv, H, D)


def h3attn_workspace_layout(B: int, Tq: int, Tkv: int, H: int, D: int = HEAD_DIM) -> dict:
    off = (ctypes.c_int64 * len(WS_FIELDS))()
    _check(lib().h3attn_workspace_layout(B, Tq, Tkv, H, D, off), "h3attn_workspace_layout")
    return dict(zip(WS_FIELDS, list(off)))


def new_workspace(B: int, Tq: int, Tkv: int, H: int, device="cuda"):
    """A uint8 device tensor of h3attn_workspace_bytes (PyTorch allocations are 512-byte aligned)."""
    import torch
    n = h3attn_workspace_bytes(B, Tq, Tkv, H)
    if n == 0:
        raise H3AttnError(ERR_INVALID_ARG, "h3attn_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def h3attn_quantize_qkv(q, k, v, ws, stream=None):
    B, Tq, H, D = q.shape
    Tkv = k.shape[1]
    wp, wb = _ptr_bytes(ws)
    vq, vk, vv = _view(q), _view(k), _view(v)
    _check(lib().h3attn_quantize_qkv(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), B, Tq, Tkv, H, D, wp, wb,
                                     _stream(stream)), "h3attn_quantize_qkv")


def h3attn_attend(ws, B: int, Tq: int, Tkv: int, H: int, softmax_scale: float, out, stream=None, D: int = HEAD_DIM):
    wp, wb = _ptr_bytes(ws)
    vo = _view(out)
    _check(lib().h3attn_attend(wp, wb, B, Tq, Tkv, H, D, softmax_scale, ctypes.byref(vo), _stream(stream)),
           "h3attn_attend")


def h3attn_forward_ex(q, k, v, softmax_scale: float, out, ws, stream=None):
    B, Tq, H, D = q.shape
    Tkv = k.shape[1]
    wp, wb = _ptr_bytes(ws)
    vq, vk, vv, vo = _view(q), _view(k), _view(v), _view(out)
    _check(lib().h3attn_forward_ex(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), B, Tq, Tkv, H, D,
                                   softmax_scale, ctypes.byref(vo), wp, wb, _stream(stream)), "h3attn_forward_ex")


def h3attn_forward(q, k, v, softmax_scale: float, out, ws, stream=None):
    """Self-attention: q, k, v and out are [B, T, H, 128] BF16 views (out may be a view of [B, T, H*128])."""
    B, T, H, D = q.shape
    wp, wb = _ptr_bytes(ws)
    vq, vk, vv, vo = _view(q), _view(k), _view(v), _view(out)
    _check(lib().h3attn_forward(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), B, T, H, D, softmax_scale,
                                ctypes.byref(vo), wp, wb, _stream(stream)), "h3attn_forward")


def _table(t, n: int, where: str) -> int:
    """Device pointer of a contiguous FP32 CUDA tensor with n elements."""
    import torch
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or t.numel() != n:
        raise ValueError(f"{where}: expected a contiguous float32 CUDA tensor of {n} elements")
    return t.data_ptr()


def _norm_rope(nr: dict, Tq: int, Tkv: int, D: int) -> _NormRope:
    """nr: gamma_q, gamma_k [D]; cos_q, sin_q [Tq, D/2]; cos_k, sin_k [Tkv, D/2] (FP32 CUDA); eps."""
    sizes = dict(gamma_q=D, gamma_k=D, cos_q=Tq * D // 2, sin_q=Tq * D // 2, cos_k=Tkv * D // 2,
                 sin_k=Tkv * D // 2)
    return _NormRope(*(_table(nr[f], sizes[f], f) for f in NORM_ROPE_FIELDS), float(nr["eps"]))


def h3attn_quantize_qkv_norm_rope(q, k, v, nr: dict, ws, stream=None):
    """h3attn_quantize_qkv with the Q/K RMSNorm + RoPE applied as the rows are loaded."""
    B, Tq, H, D = q.shape
    Tkv = k.shape[1]
    wp, wb = _ptr_bytes(ws)
    vq, vk, vv = _view(q), _view(k), _view(v)
    n = _norm_rope(nr, Tq, Tkv, D)
    _check(lib().h3attn_quantize_qkv_norm_rope(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), B, Tq, Tkv, H,
                                               D, ctypes.byref(n), wp, wb, _stream(stream)),
           "h3attn_quantize_qkv_norm_rope")


def h3attn_forward_norm_rope(q, k, v, softmax_scale: float, nr: dict, out, ws, stream=None):
    """Quantize (with the Q/K RMSNorm + RoPE) + attend."""
    B, Tq, H, D = q.shape
    Tkv = k.shape[1]
    wp, wb = _ptr_bytes(ws)
    vq, vk, vv, vo = _view(q), _view(k), _view(v), _view(out)
    n = _norm_rope(nr, Tq, Tkv, D)
    _check(lib().h3attn_forward_norm_rope(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), B, Tq, Tkv, H, D,
                                          softmax_scale, ctypes.byref(n), ctypes.byref(vo), wp, wb, _stream(stream)),
           "h3attn_forward_norm_rope")


def h3attn_norm_rope(x, gamma, cos_tab, sin_tab, eps: float, out, stream=None):
    """The separate RMSNorm + RoPE pass: x, out [B, T, H, 128] BF16 views (out may be x)."""
    B, T, H, D = x.shape
    vx, vo = _view(x), _view(out)
    _check(lib().h3attn_norm_rope(ctypes.byref(vx), B, T, H, D, _table(gamma, D, "gamma"),
                                  _table(cos_tab, T * D // 2, "cos"), _table(sin_tab, T * D // 2, "sin"), eps,
                                  ctypes.byref(vo), _stream(stream)), "h3attn_norm_rope")


def h3attn_forward_host_bytes(B: int, Tq: int, Tkv: int, H: int, heads_per_group: int, D: int = HEAD_DIM) -> int:
    return lib().h3attn_forward_host_bytes(B, Tq, Tkv, H, D, heads_per_group)


def h3attn_forward_host_groups(H: int, heads_per_group: int) -> list:
    """First head of every head group of h3attn_forward_host, then H."""
    n = lib().h3attn_forward_host_groups(H, heads_per_group, None)
    if n == 0:
        raise H3AttnError(ERR_INVALID_ARG, "h3attn_forward_host_groups")
    buf = (ctypes.c_int * (n + 1))()
    lib().h3attn_forward_host_groups(H, heads_per_group, buf)
    return list(buf)


def new_host_buffer(B: int, Tq: int, Tkv: int, H: int, heads_per_group: int, device="cuda"):
    """Device buffer for h3attn_forward_host (1024-byte aligned: the allocation is rounded up and sliced)."""
    import torch
    n = h3attn_forward_host_bytes(B, Tq, Tkv, H, heads_per_group)
    if n == 0:
        raise H3AttnError(ERR_INVALID_ARG, "h3attn_forward_host_bytes")
    raw = torch.empty(n + 1024, dtype=torch.uint8, device=device)
    skip = (-raw.data_ptr()) % 1024
    return raw[skip:skip + n]


def h3attn_forward_host(q, k, v, softmax_scale: float, out, dev_buf, heads_per_group: int, stream=None):
    """Forward pass from host q, k, v ([B, T, H, 128] BF16 CPU tensors, pinned for overlap) to a host
    out view; dev_buf from new_host_buffer with the same sizes and heads_per_group."""
    B, Tq, H, D = q.shape
    Tkv = k.shape[1]
    wp, wb = _ptr_bytes(dev_buf)
    vq, vk, vv, vo = _view(q), _view(k), _view(v), _view(out)
    _check(lib().h3attn_forward_host(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), B, Tq, Tkv, H, D,
                                     softmax_scale, ctypes.byref(vo), heads_per_group, wp, wb, _stream(stream)),
           "h3attn_forward_host")


def h3attn_forward_host_check_status(dev_buf, B: int, Tq: int, Tkv: int, H: int, heads_per_group: int,
                                     stream=None, D: int = HEAD_DIM) -> int:
    return lib().h3attn_forward_host_check_status(dev_buf.data_ptr(), B, Tq, Tkv, H, D, heads_per_group,
                                                  _stream(stream))


def h3attn_debug_forward_host_timeout(q, k, v, softmax_scale: float, out, dev_buf, heads_per_group: int,
                                      fail_group: int, wait_limit_ns: int, stream=None):
    """h3attn_forward_host with head group fail_group's waits bounded and withheld (test hook)."""
    B, Tq, H, D = q.shape
    Tkv = k.shape[1]
    wp, wb = _ptr_bytes(dev_buf)
    vq, vk, vv, vo = _view(q), _view(k), _view(v), _view(out)
    _check(lib().h3attn_debug_forward_host_timeout(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), B, Tq, Tkv,
                                                   H, D, softmax_scale, ctypes.byref(vo), heads_per_group, wp, wb,
                                                   fail_group, int(wait_limit_ns), _stream(stream)),
           "h3attn_debug_forward_host_timeout")


STATIC_WS_BYTES = 64 << 20  # H3ATTN_STATIC_WS_BYTES (the tests compare it with the loaded library's value)


def h3attn_static_workspace_bytes() -> int:
    """Size of the library's static device array (read from the loaded library)."""
    return lib().h3attn_static_workspace_bytes()


def h3attn_static_check_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the static array's sticky status word."""
    return lib().h3attn_static_check_status(_stream(stream))


def h3attn_debug_static_attend_timeout(B: int, Tq: int, Tkv: int, H: int, softmax_scale: float, out,
                                       wait_limit_ns: int, stream=None, D: int = HEAD_DIM):
    """The timeout test hook run on the static array (after an h3attn_forward_static of the same sizes)."""
    vo = _view(out)
    _check(lib().h3attn_debug_static_attend_timeout(B, Tq, Tkv, H, D, softmax_scale, ctypes.byref(vo),
                                                    int(wait_limit_ns), _stream(stream)),
           "h3attn_debug_static_attend_timeout")


def h3attn_forward_static(q, k, v, softmax_scale: float, out, stream=None):
    """Forward pass without a caller workspace: the library's static 64 MiB device array
    is used instead (for callers that cannot allocate device memory).  The first call on
    a device should come before any stream capture; calls whose GPU work overlaps race."""
    B, Tq, H, D = q.shape
    Tkv = k.shape[1]
    vq, vk, vv, vo = _view(q), _view(k), _view(v), _view(out)
    _check(lib().h3attn_forward_static(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), B, Tq, Tkv, H, D,
                                       softmax_scale, ctypes.byref(vo), _stream(stream)), "h3attn_forward_static")


def h3attn_check_status(ws, stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return lib().h3attn_check_status(ws.data_ptr(), _stream(stream))


def h3attn_debug_qk_scores(ws, B: int, Tq: int, Tkv: int, H: int, b: int, h: int, qt: int, kt: int, out,
                           stream=None, D: int = HEAD_DIM):
    """Exact INT32 QK^T tile (128 x 128) into the int32 device tensor `out`."""
    wp, wb = _ptr_bytes(ws)
    _check(lib().h3attn_debug_qk_scores(wp, wb, B, Tq, Tkv, H, D, b, h, qt, kt, out.data_ptr(), _stream(stream)),
           "h3attn_debug_qk_scores")


TRACE_EVENTS = ("s_ready", "a_pub", "p_done", "qk_issue", "pv_issue", "o_corrected", "k_full", "probs",
                "pv_done", "s_free", "ld", "max", "p_free", "pv_p", "pv_o", "turn")


def h3attn_debug_attend_trace(ws, B: int, Tq: int, Tkv: int, H: int, softmax_scale: float, out, trace_block: int,
                              stream=None, D: int = HEAD_DIM):
    """h3attn_attend with a clock64 timeline of one CTA; returns {event: int64 [2, nkv]} (0 = not recorded)."""
    import torch
    nkv = -(-Tkv // TILE)
    tr = torch.zeros(len(TRACE_EVENTS) * 2 * nkv, dtype=torch.int64, device=out.device)
    wp, wb = _ptr_bytes(ws)
    vo = _view(out)
    _check(lib().h3attn_debug_attend_trace(wp, wb, B, Tq, Tkv, H, D, softmax_scale, ctypes.byref(vo), trace_block,
                                           tr.data_ptr(), _stream(stream)), "h3attn_debug_attend_trace")
    t = tr.view(len(TRACE_EVENTS), 2, nkv).cpu()
    return {name: t[i] for i, name in enumerate(TRACE_EVENTS)}


def h3attn_debug_attend_timeout(ws, B: int, Tq: int, Tkv: int, H: int, softmax_scale: float, out,
                                wait_limit_ns: int, stream=None, D: int = HEAD_DIM):
    """h3attn_attend with the correction's O-ready arrivals withheld and every wait bounded by
    wait_limit_ns: the launch ends with H3ATTN_ERR_TIMEOUT in the workspace status word."""
    wp, wb = _ptr_bytes(ws)
    vo = _view(out)
    _check(lib().h3attn_debug_attend_timeout(wp, wb, B, Tq, Tkv, H, D, softmax_scale, ctypes.byref(vo),
                                             int(wait_limit_ns), _stream(stream)), "h3attn_debug_attend_timeout")


def workspace_views(ws, B: int, Tq: int, Tkv: int, H: int) -> dict:
    """Views of the workspace fields as stored (no copies, no conversions): q8/k8 are the
    INT8 words held as BF16 values (torch.bfloat16; compare their bit patterns)."""
    import torch
    off = h3attn_workspace_layout(B, Tq, Tkv, H)
    Tqp, Tkp = -(-Tq // TILE) * TILE, -(-Tkv // TILE) * TILE

    def sl(name, n, dtype, shape):
        nb = n * torch.tensor([], dtype=dtype).element_size()
        return ws[off[name]:off[name] + nb].view(dtype).view(shape)

    BH = B * H
    return dict(
        q8=sl("q8", BH * Tqp * 128, torch.bfloat16, (B, H, Tqp, 128)),
        k8=sl("k8", BH * Tkp * 128, torch.bfloat16, (B, H, Tkp, 128)),
        v8t=sl("v8t", BH * 128 * Tkp, torch.uint8, (B, H, 128, Tkp)),
        sq=sl("sq", BH * (Tqp // Q_GROUP), torch.float32, (B, H, Tqp // Q_GROUP)),
        sk=sl("sk", BH * (Tkp // K_GROUP), torch.float32, (B, H, Tkp // K_GROUP)),
        km=sl("km", BH * 128, torch.float32, (B, H, 128)),
        sv=sl("sv", BH * 128, torch.float32, (B, H, 128)),
    )

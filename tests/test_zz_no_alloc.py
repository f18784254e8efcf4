"""The workspace-free forward pass, h3attn_forward_static.

Some callers cannot allocate device memory: a host application that owns the
device allocator and gives this library no way to request memory through a C
interface, or a runtime whose rules forbid device allocation after start-up.
For them the library serves the workspace from a static device array of its
own.  These tests call that entry point through the C ABI several times in a
row on different shapes, a larger one before smaller ragged ones, and require
the bytes of the entry point that takes a caller workspace: both run the same
kernels, so the outputs must be identical, and contents left in the shared
array by an earlier, larger call must not leak into a later one.  The file runs
last so that a failure here leaves every other result in place; it needs
nothing from them and passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import quantized_attention_video_b200 as h3

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_attention_video_b200 import build
    build.build()
    h3.lib()


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _inputs(w):
    x = synth.make_inputs(w)
    return _dev(x["q"]), _dev(x["k"]), _dev(x["v"])


def _static_call(w, q, k, v, out):
    """h3attn_forward_static through the C ABI (ctypes), on the current stream."""
    vq, vk, vv, vo = h3._view(q), h3._view(k), h3._view(v), h3._view(out)
    return h3.lib().h3attn_forward_static(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), w.B, w.Tq, w.Tkv,
                                          w.H, w.D, w.scale, ctypes.byref(vo),
                                          torch.cuda.current_stream().cuda_stream)


def _workspace_forward(w, q, k, v):
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    ref = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device="cuda")
    h3.h3attn_forward_ex(q, k, v, w.scale, ref, ws)
    assert h3.h3attn_check_status(ws) == h3.OK
    return ref


def _same_bytes(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_the_array_size_is_the_library_s():
    assert h3.h3attn_static_workspace_bytes() == h3.STATIC_WS_BYTES == 64 << 20


def test_static_forward_matches_workspace_forward_larger_call_first():
    cases = [synth.WORKLOADS["selfattn_h8_t4096"],                          # the largest first
             synth.Workload("static_ragged", 1, 300, 457, 3, 128, "k_offset", 6101),  # then smaller, ragged
             synth.Workload("static_ragged_b2", 2, 77, 129, 2, 128, "rmsnorm", 6102),
             synth.WORKLOADS["fixed_q128_kv192"]]
    inputs = [_inputs(w) for w in cases]
    refs = [_workspace_forward(w, *t) for w, t in zip(cases, inputs)]
    outs = []
    for w, (q, k, v) in zip(cases, inputs):  # calls in a row on the shared static array
        assert h3.h3attn_workspace_bytes(w.B, w.Tq, w.Tkv, w.H) <= h3.STATIC_WS_BYTES
        out = torch.full((w.B, w.Tq, w.H, w.D), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _static_call(w, q, k, v, out) == h3.OK
        outs.append(out)
    assert h3.h3attn_static_check_status() == h3.OK
    for w, out, ref in zip(cases, outs, refs):
        assert _same_bytes(out, ref), w.name


def _largest_fitting_T():
    """Largest T (B = 1, H = 1, Tq = Tkv = T) whose workspace fits the static array."""
    lo, hi = 1, 1 << 20
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if h3.h3attn_workspace_bytes(1, mid, mid, 1) <= h3.STATIC_WS_BYTES:
            lo = mid
        else:
            hi = mid - 1
    return lo


def test_the_largest_fitting_shape_runs_and_one_token_more_is_rejected():
    T = _largest_fitting_T()
    assert h3.h3attn_workspace_bytes(1, T, T, 1) <= h3.STATIC_WS_BYTES < h3.h3attn_workspace_bytes(1, T + 1, T + 1, 1)
    w = synth.Workload("static_max", 1, T, T, 1, 128, "normal", 6103)
    q, k, v = _inputs(w)
    ref = _workspace_forward(w, q, k, v)
    out = torch.empty_like(ref)
    assert _static_call(w, q, k, v, out) == h3.OK
    assert h3.h3attn_static_check_status() == h3.OK
    assert _same_bytes(out, ref)
    # one token past the limit: rejected before anything is read or enqueued
    w1 = synth.Workload("static_max_plus_1", 1, T + 1, T + 1, 1, 128, "normal", 6104)
    small = torch.empty(1, 8, 1, 128, dtype=torch.bfloat16, device="cuda")
    vs = h3._View(small.data_ptr(), 8 * 128, 128, 128)
    st = h3.lib().h3attn_forward_static(ctypes.byref(vs), ctypes.byref(vs), ctypes.byref(vs), w1.B, w1.Tq, w1.Tkv,
                                        w1.H, w1.D, w1.scale, ctypes.byref(vs), None)
    assert st == h3.ERR_WORKSPACE


def test_static_forward_rejects_shapes_beyond_its_array():
    w = synth.WORKLOADS["h3_t37810_h32"]
    assert h3.h3attn_workspace_bytes(w.B, w.Tq, w.Tkv, w.H) > h3.STATIC_WS_BYTES
    small = torch.empty(1, 8, 1, 128, dtype=torch.bfloat16, device="cuda")
    # the size check comes first: nothing is read or enqueued for these pointers
    vq = h3._View(small.data_ptr(), w.Tq * w.H * w.D, w.H * w.D, w.D)
    vo = h3._View(small.data_ptr(), w.Tq * w.H * w.D, w.H * w.D, w.D)
    st = h3.lib().h3attn_forward_static(ctypes.byref(vq), ctypes.byref(vq), ctypes.byref(vq), w.B, w.Tq, w.Tkv,
                                        w.H, w.D, w.scale, ctypes.byref(vo), None)
    assert st == h3.ERR_WORKSPACE


def test_a_device_timeout_on_the_static_array_is_reported_and_the_array_recovers():
    """A bounded wait that runs out on the static array (the test hook withholds an
    arrival; no fault) is read back by h3attn_static_check_status, which allocates
    nothing; a later static call gives the normal bytes again."""
    w = synth.WORKLOADS["fixed_q128_kv192"]
    q, k, v = _inputs(w)
    ref = _workspace_forward(w, q, k, v)
    out = torch.empty_like(ref)
    assert _static_call(w, q, k, v, out) == h3.OK
    assert h3.h3attn_static_check_status() == h3.OK
    h3.h3attn_debug_static_attend_timeout(w.B, w.Tq, w.Tkv, w.H, w.scale, out, LIMIT_NS)
    assert h3.h3attn_static_check_status() == h3.ERR_TIMEOUT
    assert h3.h3attn_static_check_status() == h3.OK
    again = torch.empty_like(ref)
    assert _static_call(w, q, k, v, again) == h3.OK
    assert h3.h3attn_static_check_status() == h3.OK
    assert _same_bytes(again, ref)

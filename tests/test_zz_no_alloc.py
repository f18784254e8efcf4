"""The workspace-free forward pass, h3attn_forward_static.

Some callers cannot allocate device memory: a host application that owns the
device allocator and gives this library no way to request memory through a C
interface, or a runtime whose rules forbid device allocation after start-up.
For them the library serves the workspace from a static device array of its
own (64 MiB).  These tests call that entry point through the C ABI, twice in a
row on two different shapes, and compare each output with the entry point that
takes a caller workspace, run on the same inputs.  The file runs last so that a
failure here leaves every other result in place; it needs nothing from them.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import quantized_attention_video_b200 as h3

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_attention_video_b200 import build
    build.build()
    h3.lib()


def _inputs(name):
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w)

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)

    return w, dev(x["q"]), dev(x["k"]), dev(x["v"])


def _static_call(w, q, k, v, out):
    """h3attn_forward_static through the C ABI (ctypes), on the current stream."""
    vq, vk, vv, vo = h3._view(q), h3._view(k), h3._view(v), h3._view(out)
    return h3.lib().h3attn_forward_static(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), w.B, w.Tq, w.Tkv,
                                          w.H, w.D, w.scale, ctypes.byref(vo),
                                          torch.cuda.current_stream().cuda_stream)


def _compare(got, ref, what):
    g = got.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all(), what
    err = np.abs(g - r).max()
    rel = np.linalg.norm(g - r) / np.linalg.norm(r)
    assert err <= MAX_ABS, f"{what}: max-abs {err:.3e}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e}"


def test_static_forward_matches_workspace_forward_twice():
    cases = [_inputs("fixed_q128_kv192"), _inputs("selfattn_h8_t4096")]
    refs = []
    for w, q, k, v in cases:
        assert h3.h3attn_workspace_bytes(w.B, w.Tq, w.Tkv, w.H) <= h3.STATIC_WS_BYTES
        ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
        ref = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device="cuda")
        h3.h3attn_forward_ex(q, k, v, w.scale, ref, ws)
        assert h3.h3attn_check_status(ws) == h3.OK
        refs.append(ref)
    outs = []
    for w, q, k, v in cases:  # two calls in a row on the shared static array
        out = torch.full((w.B, w.Tq, w.H, w.D), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _static_call(w, q, k, v, out) == h3.OK
        outs.append(out)
    torch.cuda.synchronize()
    for (w, _, _, _), out, ref in zip(cases, outs, refs):
        _compare(out, ref, w.name)


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

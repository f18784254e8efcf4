"""h3attn_forward_host: the forward pass from host buffers, pipelined by head groups,
gives the same bytes as the device forward pass on all heads at once (heads are
independent problems: every statistic, scale and softmax is per (b, h))."""
import numpy as np
import pytest
import torch

import synth
import quantized_attention_video_b200 as h3

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_attention_video_b200 import build
    build.build()
    h3.lib()


def _host(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()


def _device_reference(q, k, v, scale):
    """Device forward pass of all heads at once."""
    B, Tq, H, D = q.shape
    Tkv = k.shape[1]
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty(B, Tq, H, D, dtype=torch.bfloat16, device="cuda")
    ws = h3.new_workspace(B, Tq, Tkv, H)
    h3.h3attn_forward_ex(dq, dk, dv, scale, out, ws)
    assert h3.h3attn_check_status(ws) == h3.OK
    return out.cpu()


def _run_host(q, k, v, scale, out, g):
    B, Tq, H, D = q.shape
    Tkv = k.shape[1]
    buf = h3.new_host_buffer(B, Tq, Tkv, H, g)
    h3.h3attn_forward_host(q, k, v, scale, out, buf, g)
    torch.cuda.current_stream().synchronize()
    assert h3.h3attn_forward_host_check_status(buf, B, Tq, Tkv, H, g) == h3.OK


@pytest.mark.parametrize("name, g", [("selfattn_h8_t4096", 3), ("selfattn_h8_t4096", 8), ("fixed_q128_kv192", 1)])
def test_host_pipeline_matches_device_forward(name, g):
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w)
    q, k, v = _host(x["q"]), _host(x["k"]), _host(x["v"])
    ref = _device_reference(q, k, v, w.scale)
    out = torch.full((w.B, w.Tq, w.H, w.D), 3.0, dtype=torch.bfloat16).pin_memory()
    _run_host(q, k, v, w.scale, out, g)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_host_pipeline_packed_qkv_into_token_major_output():
    """Packed [B, T, 3, H, D] host input and [B, T, H*D] host output, B = 2, ragged T."""
    B, T, H, D = 2, 300, 4, 128
    w = synth.Workload("host_packed", B, T, T, H, D, "normal", 515)
    x = synth.make_inputs(w)
    packed = torch.empty(B, T, 3, H, D, dtype=torch.bfloat16).pin_memory()
    for i, n in enumerate(("q", "k", "v")):
        packed[:, :, i] = torch.from_numpy(np.ascontiguousarray(x[n]).view(np.int16)).view(torch.bfloat16)
    q, k, v = packed[:, :, 0], packed[:, :, 1], packed[:, :, 2]
    ref = _device_reference(q.contiguous(), k.contiguous(), v.contiguous(), w.scale)
    out = torch.zeros(B, T, H * D, dtype=torch.bfloat16).pin_memory()
    _run_host(q, k, v, w.scale, out.view(B, T, H, D), 3)
    assert torch.equal(out.view(B, T, H, D).view(torch.int16), ref.view(torch.int16))


def test_host_pipeline_head_major_layout():
    """Host tensors stored [B, H, T, D] (heads not adjacent within a token): one copy per head."""
    w = synth.Workload("host_hmajor", 1, 777, 777, 5, 128, "k_offset", 99)
    x = synth.make_inputs(w)
    def head_major(a):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        return t.permute(0, 2, 1, 3).contiguous().pin_memory().permute(0, 2, 1, 3)  # [B, T, H, D] view
    q, k, v = head_major(x["q"]), head_major(x["k"]), head_major(x["v"])
    assert q.stride(2) != 128
    ref = _device_reference(q.contiguous(), k.contiguous(), v.contiguous(), w.scale)
    out = torch.empty(1, 5, 777, 128, dtype=torch.bfloat16).pin_memory().permute(0, 2, 1, 3)
    _run_host(q, k, v, w.scale, out, 2)
    assert torch.equal(out.contiguous().view(torch.int16), ref.view(torch.int16))

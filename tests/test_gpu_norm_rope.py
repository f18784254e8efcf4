"""GPU parity of the Q/K RMSNorm + RoPE preparation against the CPU oracle.

The step is the Q/K normalization and RoPE of the H3 block ("H3 Performance
Roadmap": "Norm and RoPE" in the representative block table; Component 2,
item 1: applied where the attention consumes Q and K).  Bar:
  * the separate pass (h3attn_norm_rope): BF16 output bit-exact;
  * the fused preparation (h3attn_quantize_qkv_norm_rope): INT8 Q/K words, FP8 V
    words, every scale and the K means bit-exact against the oracle's
    qk_norm_rope + quantize, and equal to the separate pass followed by the plain
    preparation;
  * the forward output: max-abs <= 1e-2 and relative L2 <= 2e-3 (as the plain path).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_attention_video_b200 as h3
from test_gpu_parity import EPOCH, bits, check_quantized, compare_out, new_out, sample_rows, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_attention_video_b200 import build
    build.build()
    h3.lib()


def dev_params(nr: dict) -> dict:
    out = {n: torch.from_numpy(np.ascontiguousarray(nr[n], dtype=np.float32)).cuda() for n in h3.NORM_ROPE_FIELDS}
    out["eps"] = nr["eps"]
    return out


def workload(B, Tq, Tkv, H, seed):
    return synth.Workload(f"nr_{B}_{Tq}_{Tkv}_{H}", B, Tq, Tkv, H, 128, "normal", seed, norm_rope=True)


def test_separate_pass_bit_exact_strided_and_in_place():
    w = synth.WORKLOADS["nr_h4_t1100"]
    nr = synth.norm_rope_params(w)
    dn = dev_params(nr)
    # a packed [B, T, 3, H, D] buffer: normalize its K slot through the strided view
    pw = synth.Workload("nr_packed", 1, 1100, 1100, 4, 128, "normal", 1101, packed=True)
    x = synth.make_inputs(pw)
    d = upload(x, pw)
    ref = oracle.qk_norm_rope(x["k"], nr["gamma_k"], nr["eps"], nr["cos_k"], nr["sin_k"])
    out = torch.empty(1, 1100, 4, 128, dtype=torch.bfloat16, device="cuda")
    h3.h3attn_norm_rope(d["k"], dn["gamma_k"], dn["cos_k"], dn["sin_k"], nr["eps"], out)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out), ref)
    # in place on the packed view; the Q and V slots stay untouched
    q_before, v_before = bits(d["q"]), bits(d["v"])
    h3.h3attn_norm_rope(d["k"], dn["gamma_k"], dn["cos_k"], dn["sin_k"], nr["eps"], d["k"])
    torch.cuda.synchronize()
    assert np.array_equal(bits(d["k"]), ref)
    assert np.array_equal(bits(d["q"]), q_before) and np.array_equal(bits(d["v"]), v_before)


FUSED = [(1, 1100, 1100, 4), (1, 200, 300, 2), (2, 129, 1000, 1), (1, 1, 1, 1), (1, 700, 130, 3)]


@pytest.mark.parametrize("B,Tq,Tkv,H", FUSED)
def test_fused_preparation_and_forward(B, Tq, Tkv, H):
    w = synth.WORKLOADS["nr_h4_t1100"] if (B, Tq, Tkv, H) == (1, 1100, 1100, 4) else workload(B, Tq, Tkv, H,
                                                                                           3000 + Tq + 7 * Tkv)
    x = synth.make_inputs(w)
    nr = synth.norm_rope_params(w)
    z = oracle.quantize_norm_rope(x["q"], x["k"], x["v"], nr)
    d = upload(x, w)
    dn = dev_params(nr)
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    out, out4 = new_out(w)
    h3.h3attn_forward_norm_rope(d["q"], d["k"], d["v"], w.scale, dn, out4, ws)
    assert h3.h3attn_check_status(ws) == h3.OK
    check_quantized(ws, z, w)
    compare_out(bits(out4), oracle.attend_all(z, w.scale, EPOCH), w.name)


def test_fused_reads_packed_strided_views():
    # raw Q/K/V read in place from one packed [B, T, 3, H, D] buffer, output into [B, T, H*D]
    w = synth.Workload("nr_packed_b2", 2, 300, 300, 3, 128, "normal", 4301, packed=True, norm_rope=True)
    x = synth.make_inputs(w)
    nr = synth.norm_rope_params(w)
    z = oracle.quantize_norm_rope(x["q"], x["k"], x["v"], nr)
    d = upload(x, w)
    dn = dev_params(nr)
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    out, out4 = new_out(w)
    h3.h3attn_forward_norm_rope(d["q"], d["k"], d["v"], w.scale, dn, out4, ws)
    assert h3.h3attn_check_status(ws) == h3.OK
    check_quantized(ws, z, w)
    compare_out(bits(out4), oracle.attend_all(z, w.scale, EPOCH), w.name)
    assert out.shape == (w.B, w.Tq, w.H * w.D) and out.is_contiguous()


def test_bench_shape_fused_equals_oracle_and_separate_pass():
    w = synth.WORKLOADS["h3_t37810_h32_nr"]
    x = synth.make_inputs(w)
    nr = synth.norm_rope_params(w)
    z = oracle.quantize_norm_rope(x["q"], x["k"], x["v"], nr)
    d = upload(x, w)
    dn = dev_params(nr)
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    out, out4 = new_out(w)
    h3.h3attn_forward_norm_rope(d["q"], d["k"], d["v"], w.scale, dn, out4, ws)
    assert h3.h3attn_check_status(ws) == h3.OK
    check_quantized(ws, z, w)
    rows = sample_rows(w, 1, seed=w.seed)
    ref, _, _ = oracle.attend_rows(z, w.scale, EPOCH, rows)
    compare_out(bits(out4)[rows[:, 0], rows[:, 2], rows[:, 1]], ref, w.name)
    # the separate pass + the plain preparation writes the same workspace words
    qn = torch.empty_like(d["q"])
    kn = torch.empty_like(d["k"])
    h3.h3attn_norm_rope(d["q"], dn["gamma_q"], dn["cos_q"], dn["sin_q"], nr["eps"], qn)
    h3.h3attn_norm_rope(d["k"], dn["gamma_k"], dn["cos_k"], dn["sin_k"], nr["eps"], kn)
    ws2 = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    h3.h3attn_quantize_qkv(qn, kn, d["v"], ws2)
    assert h3.h3attn_check_status(ws2) == h3.OK
    va = h3.workspace_views(ws, w.B, w.Tq, w.Tkv, w.H)
    vb = h3.workspace_views(ws2, w.B, w.Tq, w.Tkv, w.H)
    for f in ("q8", "k8", "v8t", "sq", "sk", "km", "sv"):
        assert np.array_equal(bits(va[f]), bits(vb[f])), f


def test_fused_forward_replays_from_a_cuda_graph():
    """The norm + RoPE forward (five launches, no host synchronisation) captured once into a
    CUDA graph replays the bytes of a direct call."""
    w = synth.WORKLOADS["nr_h4_t1100"]
    x = synth.make_inputs(w)
    nr = synth.norm_rope_params(w)
    d = upload(x, w)
    dn = dev_params(nr)
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    direct = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device="cuda")
    h3.h3attn_forward_norm_rope(d["q"], d["k"], d["v"], w.scale, dn, direct, ws)
    assert h3.h3attn_check_status(ws) == h3.OK
    out = torch.zeros_like(direct)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up on the capture stream
        h3.h3attn_forward_norm_rope(d["q"], d["k"], d["v"], w.scale, dn, out, ws)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        h3.h3attn_forward_norm_rope(d["q"], d["k"], d["v"], w.scale, dn, out, ws)
    for _ in range(20):
        out.zero_()
        g.replay()
        torch.cuda.current_stream().synchronize()
        assert torch.equal(out.view(torch.int16), direct.view(torch.int16))
    assert h3.h3attn_check_status(ws) == h3.OK

"""Failure detection on the GPU without a fault: bounded waits that run out.

The test hook h3attn_debug_attend_timeout runs the attention kernel with the
correction warpgroup's "O ready" arrivals withheld and every barrier wait
bounded by a short limit.  The first wait to run out records
H3ATTN_ERR_TIMEOUT and its wait-site id in the workspace status word and
raises its CTA's abort flag; every role drains the copies and tensor-core work
it started and returns.  Nothing faults or traps, and the same CUDA context
then runs the normal path to the same output as before: the failure side of the
no-deadlock requirement of "Phase 2B Aligned Numerical Prototype", Exactness.
"""
import time

import numpy as np
import pytest
import torch

import synth
import quantized_attention_video_b200 as h3

pytestmark = pytest.mark.gpu

# Wait-site ids of the waits that the withheld arrival leaves without a producer
# (which of them runs out first depends on when each started waiting):
SITE_K_PRODUCER, SITE_V_PRODUCER = 1, 2  # producers waiting for a free stage
SITE_PV_O_READY = 6                      # PV issuer waiting for "O ready"
SITE_QK_S_FREE = 8                       # QK issuer waiting for a free score buffer
SITE_SOFTMAX_PV = 11                     # softmax waiting for its probability buffer
SITE_CORR_PV = 13                        # correction waiting for PV of the previous tile
SITE_SOFTMAX_TURN = 10                   # softmax waiting for its MUFU turn
SMALL_SITES = {SITE_PV_O_READY, SITE_SOFTMAX_PV, SITE_CORR_PV}
LARGE_SITES = SMALL_SITES | {SITE_K_PRODUCER, SITE_V_PRODUCER, SITE_QK_S_FREE, SITE_SOFTMAX_TURN}
LIMIT_NS = 20_000_000  # 20 ms


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
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    return w, dev(x["q"]), dev(x["k"]), dev(x["v"])


def _status_words(ws):
    torch.cuda.synchronize()
    return ws[:12].cpu().numpy().view(np.int32).tolist()  # code, detail, block


@pytest.mark.parametrize("name, sites", [("fixed_q128_kv192", SMALL_SITES),
                                         ("selfattn_h8_t4096", LARGE_SITES)])
def test_withheld_arrival_times_out_and_the_context_stays_usable(name, sites):
    w, q, k, v = _inputs(name)
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    ref = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device="cuda")
    h3.h3attn_quantize_qkv(q, k, v, ws)
    h3.h3attn_attend(ws, w.B, w.Tq, w.Tkv, w.H, w.scale, ref)
    assert h3.h3attn_check_status(ws) == h3.OK

    bad = torch.zeros_like(ref)
    t0 = time.perf_counter()
    h3.h3attn_debug_attend_timeout(ws, w.B, w.Tq, w.Tkv, w.H, w.scale, bad, LIMIT_NS)
    code, detail, block = _status_words(ws)
    elapsed = time.perf_counter() - t0
    assert code == h3.ERR_TIMEOUT
    assert detail in sites
    ntq = -(-w.Tq // 128)
    assert 0 <= block < ((ntq + 1) // 2) * w.H * w.B
    assert elapsed < 5.0  # bounded: the waits gave up instead of hanging
    assert h3.h3attn_check_status(ws) == h3.ERR_TIMEOUT  # reads and clears the word
    assert h3.h3attn_check_status(ws) == h3.OK

    # the context is healthy: the normal path runs again to the same bytes
    again = torch.empty_like(ref)
    h3.h3attn_attend(ws, w.B, w.Tq, w.Tkv, w.H, w.scale, again)
    assert h3.h3attn_check_status(ws) == h3.OK
    assert torch.equal(again.view(torch.int16), ref.view(torch.int16))


def test_timeout_hook_rejects_out_of_range_limits():
    w, q, k, v = _inputs("fixed_q128_kv192")
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    out = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device="cuda")
    for bad in (0, 999_999, 3_000_000_000):
        with pytest.raises(h3.H3AttnError):
            h3.h3attn_debug_attend_timeout(ws, w.B, w.Tq, w.Tkv, w.H, w.scale, out, bad)


def test_status_is_sticky_across_later_calls():
    """A timeout recorded by one call survives later calls on the same workspace (their
    preparation does not clear it) until h3attn_check_status reads it ("Phase 2B Aligned
    Numerical Prototype", Synchronization And Safety: a failure must not be lost)."""
    w, q, k, v = _inputs("fixed_q128_kv192")
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    out = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device="cuda")
    h3.h3attn_forward_ex(q, k, v, w.scale, out, ws)
    assert h3.h3attn_check_status(ws) == h3.OK
    h3.h3attn_debug_attend_timeout(ws, w.B, w.Tq, w.Tkv, w.H, w.scale, out, LIMIT_NS)
    for _ in range(3):  # later, successful calls on the same workspace
        h3.h3attn_forward_ex(q, k, v, w.scale, out, ws)
    assert h3.h3attn_check_status(ws) == h3.ERR_TIMEOUT
    assert h3.h3attn_check_status(ws) == h3.OK


@pytest.mark.parametrize("fail_group", [0, 1, 2])
def test_host_pipeline_reports_an_early_group_timeout(fail_group):
    """h3attn_forward_host over 5 head groups of 1, 2, 2, 2 and 1 heads (two device slots
    reused in turn) with the waits of one early group withheld:
    h3attn_forward_host_check_status reports the timeout although later groups reused that
    group's slot; the heads of the other groups are those of the normal pipeline."""
    w = synth.WORKLOADS["selfattn_h8_t4096"]
    x = synth.make_inputs(w)
    host = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()
    q, k, v = host(x["q"]), host(x["k"]), host(x["v"])
    g = 2
    starts = h3.h3attn_forward_host_groups(w.H, g)
    assert starts == [0, 1, 3, 5, 7, 8]  # halved first and last groups
    buf = h3.new_host_buffer(w.B, w.Tq, w.Tkv, w.H, g)
    ref = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16).pin_memory()
    h3.h3attn_forward_host(q, k, v, w.scale, ref, buf, g)
    assert h3.h3attn_forward_host_check_status(buf, w.B, w.Tq, w.Tkv, w.H, g) == h3.OK
    out = torch.zeros_like(ref).pin_memory()
    h3.h3attn_debug_forward_host_timeout(q, k, v, w.scale, out, buf, g, fail_group, LIMIT_NS)
    assert h3.h3attn_forward_host_check_status(buf, w.B, w.Tq, w.Tkv, w.H, g) == h3.ERR_TIMEOUT
    assert h3.h3attn_forward_host_check_status(buf, w.B, w.Tq, w.Tkv, w.H, g) == h3.OK
    others = [h for h in range(w.H) if not starts[fail_group] <= h < starts[fail_group + 1]]
    assert torch.equal(out[:, :, others].view(torch.int16), ref[:, :, others].view(torch.int16))


def test_host_timeout_hook_rejects_a_group_out_of_range():
    w = synth.WORKLOADS["fixed_q128_kv192"]
    x = synth.make_inputs(w)
    host = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()
    q, k, v = host(x["q"]), host(x["k"]), host(x["v"])
    buf = h3.new_host_buffer(w.B, w.Tq, w.Tkv, w.H, 1)
    out = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16).pin_memory()
    with pytest.raises(h3.H3AttnError):
        h3.h3attn_debug_forward_host_timeout(q, k, v, w.scale, out, buf, 1, 1, LIMIT_NS)

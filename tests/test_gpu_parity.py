"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bar (per the numerical policy of "H3 Performance Roadmap", Phase 4, and the
checkpoints of "Phase 2B Aligned Numerical Prototype", Exactness):
  * INT8 Q/K words, FP8 V words, every scale and the K means: bit-exact;
  * INT32 QK^T scores: bit-exact (through the debug export, same MMA path);
  * BF16 output: max-abs <= 1e-2 and relative L2 <= 2e-3 against the oracle run
    with the kernel's 128-key softmax epoch.
Inputs are the seeded synthetic workloads of the synth module.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_attention_video_b200 as h3

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 2e-3
EPOCH = 128  # the kernel's key tile = its online-softmax epoch


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_attention_video_b200 import build
    build.build()
    h3.lib()  # raises loudly if the library is missing


def upload(x: dict, w: synth.Workload):
    """Device BF16 views for q, k, v (and the packed buffer when the workload is packed)."""
    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    if w.packed:
        buf = dev(x["packed"])
        return {"buf": buf, "q": buf[:, :, 0], "k": buf[:, :, 1], "v": buf[:, :, 2]}
    return {n: dev(x[n]) for n in ("q", "k", "v")}


def new_out(w: synth.Workload):
    if w.packed:
        o = torch.empty(w.B, w.Tq, w.H * w.D, dtype=torch.bfloat16, device="cuda")
        return o, o.view(w.B, w.Tq, w.H, w.D)
    o = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device="cuda")
    return o, o


def bits(t: torch.Tensor) -> np.ndarray:
    t = t.contiguous().cpu()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def f32_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.int32)


def int8_as_bf16_bits(a: np.ndarray) -> np.ndarray:
    """The exact BF16 encoding of integer words in [-127, 127] (the form the workspace
    stores them in): the top half of their FP32 encoding, whose low half is zero."""
    f = np.ascontiguousarray(a, dtype=np.int8).astype(np.float32).view(np.uint32)
    assert not (f & 0xFFFF).any()
    return (f >> 16).astype(np.uint16)


def check_quantized(ws, z, w):
    B, Tq, Tkv, H = w.B, w.Tq, w.Tkv, w.H
    v = h3.workspace_views(ws, B, Tq, Tkv, H)
    # the stored bit patterns of the Q/K words against the exact encoding of the
    # oracle's integers (no conversion of the GPU's words), padding +0 exactly
    q8, k8, v8t = bits(v["q8"]), bits(v["k8"]), bits(v["v8t"])
    assert np.array_equal(q8[:, :, :Tq], int8_as_bf16_bits(z["q8"])), "q8"
    assert not q8[:, :, Tq:].any()
    assert np.array_equal(k8[:, :, :Tkv], int8_as_bf16_bits(z["k8"])), "k8"
    assert not k8[:, :, Tkv:].any()
    assert np.array_equal(v8t[:, :, :, :Tkv].transpose(0, 1, 3, 2), z["v8"]), "v8"
    assert not v8t[:, :, :, Tkv:].any()
    nq, nk = z["sq"].shape[-1], z["sk"].shape[-1]
    sq, sk = bits(v["sq"]), bits(v["sk"])
    assert np.array_equal(sq[:, :, :nq], f32_bits(z["sq"])), "sq"
    assert not sq[:, :, nq:].any()
    assert np.array_equal(sk[:, :, :nk], f32_bits(z["sk"])), "sk"
    assert not sk[:, :, nk:].any()
    assert np.array_equal(bits(v["km"]), f32_bits(z["km"])), "km"
    assert np.array_equal(bits(v["sv"]), f32_bits(z["sv"])), "sv"


def compare_out(got: np.ndarray, ref: np.ndarray, what: str):
    g = oracle.bf16_decode(got).astype(np.float64)
    r = oracle.bf16_decode(ref).astype(np.float64)
    assert np.isfinite(g).all(), what
    err = np.abs(g - r)
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    assert err.max() <= MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e}"
    return err.max(), rel


def sample_tiles(ntile: int, n_random: int, rng) -> list:
    """Q tiles checked for one (b, h): the first two and the last two (the ragged tail
    among them) plus n_random distinct seeded interior tiles."""
    fixed = {t for t in (0, 1, ntile - 2, ntile - 1) if 0 <= t < ntile}
    interior = [t for t in range(ntile) if t not in fixed]
    picked = rng.choice(interior, size=min(n_random, len(interior)), replace=False) if interior else []
    return sorted(fixed | {int(t) for t in picked})


def sample_rows(w: synth.Workload, n_random: int, seed: int):
    """(b, h, i) rows of sample_tiles for every batch item and head."""
    rng = np.random.default_rng(seed)
    ntile = -(-w.Tq // 128)
    rows = []
    for b in range(w.B):
        for h in range(w.H):
            for t in sample_tiles(ntile, n_random, rng):
                for i in range(t * 128, min(w.Tq, t * 128 + 128)):
                    rows.append((b, h, i))
    return np.array(rows, dtype=np.int32)


def run_forward(w, d):
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    out, out4 = new_out(w)
    if w.Tq == w.Tkv:
        h3.h3attn_forward(d["q"], d["k"], d["v"], w.scale, out4, ws)
    else:
        h3.h3attn_forward_ex(d["q"], d["k"], d["v"], w.scale, out4, ws)
    assert h3.h3attn_check_status(ws) == h3.OK
    return ws, out, out4


# ---------------------------------------------------------------- configs ----
# Output rows compared with the oracle: every row of the first two workloads; for the
# others, every (b, h) with its first two and last two Q tiles plus 8 seeded interior
# ones (sample_tiles):
#   ragged_h16_t9453     16 heads x (11 x 128 + 109) rows        = 24,272 rows
#   h3_t37810_h32        32 heads x (11 x 128 + 50) rows         = 46,656 rows
#   h3_packed_b2_t37810  2 batch items x 32 heads x 1,458 rows   = 93,312 rows
#   h3_t74000_h32        32 heads x (11 x 128 + 16) rows         = 45,568 rows
FULL = ["fixed_q128_kv192", "selfattn_h8_t4096"]
SAMPLED = {"ragged_h16_t9453": 8, "h3_t37810_h32": 8, "h3_packed_b2_t37810": 8, "h3_t74000_h32": 8}
SAMPLED_ROWS = {"ragged_h16_t9453": 24272, "h3_t37810_h32": 46656, "h3_packed_b2_t37810": 93312,
                "h3_t74000_h32": 45568}


@pytest.mark.parametrize("name", FULL + list(SAMPLED))
def test_workload_parity(name):
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w)
    z = oracle.quantize(x["q"], x["k"], x["v"])
    d = upload(x, w)
    ws, out, out4 = run_forward(w, d)
    check_quantized(ws, z, w)
    got = bits(out4)  # [B, T, H, D]
    if name in FULL:
        ref = oracle.attend_all(z, w.scale, EPOCH)
        compare_out(got, ref, name)
    else:
        rows = sample_rows(w, SAMPLED[name], seed=w.seed)
        assert len(rows) == SAMPLED_ROWS[name]
        ref, _, _ = oracle.attend_rows(z, w.scale, EPOCH, rows)
        compare_out(got[rows[:, 0], rows[:, 2], rows[:, 1]], ref, name)
    if w.packed:
        # the output is the token-major [B, T, H*D] buffer itself
        assert out.shape == (w.B, w.Tq, w.H * w.D) and out.is_contiguous()


@pytest.mark.parametrize("name", FULL + list(SAMPLED))
def test_qk_scores_bit_exact(name):
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w)
    z = oracle.quantize(x["q"], x["k"], x["v"])
    d = upload(x, w)
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    h3.h3attn_quantize_qkv(d["q"], d["k"], d["v"], ws)
    nq, nk = -(-w.Tq // 128), -(-w.Tkv // 128)
    rng = np.random.default_rng(7)
    tiles = {(0, 0, 0, 0), (w.B - 1, w.H - 1, nq - 1, nk - 1)}
    while len(tiles) < min(16, w.B * w.H * nq * nk):
        tiles.add((int(rng.integers(w.B)), int(rng.integers(w.H)), int(rng.integers(nq)), int(rng.integers(nk))))
    buf = torch.empty(128, 128, dtype=torch.int32, device="cuda")
    for (b, h, qt, kt) in sorted(tiles):
        h3.h3attn_debug_qk_scores(ws, w.B, w.Tq, w.Tkv, w.H, b, h, qt, kt, buf)
        g = buf.cpu().numpy()
        ni, nj = min(128, w.Tq - qt * 128), min(128, w.Tkv - kt * 128)
        ref = oracle.scores(z, b, h, qt * 128, ni, kt * 128, nj)
        assert np.array_equal(g[:ni, :nj], ref), (b, h, qt, kt)
        # padded rows / keys are zero words, so their scores are exactly 0
        assert not g[ni:].any() and not g[:, nj:].any()
    assert h3.h3attn_check_status(ws) == h3.OK


# ------------------------------------------------------------- edge cases ----
EDGE = [(1, 1, 1, 1), (1, 1, 200, 1), (1, 200, 1, 1), (1, 127, 129, 2), (2, 129, 127, 1), (1, 255, 256, 1),
        (1, 257, 300, 3), (3, 64, 64, 2), (1, 384, 640, 1), (1, 130, 1000, 2)]


@pytest.mark.parametrize("B,Tq,Tkv,H", EDGE)
def test_edge_shapes(B, Tq, Tkv, H):
    w = synth.Workload(f"edge_{B}_{Tq}_{Tkv}_{H}", B, Tq, Tkv, H, 128, "normal", 1000 + Tq * 7 + Tkv)
    x = synth.make_inputs(w)
    z = oracle.quantize(x["q"], x["k"], x["v"])
    d = upload(x, w)
    ws, out, out4 = run_forward(w, d)
    check_quantized(ws, z, w)
    compare_out(bits(out4), oracle.attend_all(z, w.scale, EPOCH), w.name)


def test_degenerate_zero_inputs():
    w = synth.Workload("zeros", 1, 200, 300, 2, 128, "normal", 5)
    x = synth.make_inputs(w)
    x["q"][:, :, 0] = 0          # head 0: all-zero Q -> uniform softmax
    x["k"][:, :, 1] = 0          # head 1: all-zero K -> zero scores
    x["v"][:, 50:, 1, :64] = 0   # some V channels zero after token 50
    x["v"][:, :, 0, 100:] = 0    # V channels that are zero everywhere -> zero scale, zero output
    z = oracle.quantize(x["q"], x["k"], x["v"])
    d = upload(x, w)
    ws, out, out4 = run_forward(w, d)
    check_quantized(ws, z, w)
    got = bits(out4)
    compare_out(got, oracle.attend_all(z, w.scale, EPOCH), "zeros")
    assert not got[:, :, 0, 100:].any()


def test_output_strides_and_untouched_padding():
    """Output written through a strided view; rows and channels outside it stay untouched."""
    w = synth.Workload("strided_out", 1, 300, 300, 2, 128, "normal", 77)
    x = synth.make_inputs(w)
    z = oracle.quantize(x["q"], x["k"], x["v"])
    d = upload(x, w)
    big = torch.full((1, 300, 2, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    view = big[:, :, :, 64:192]
    ws = h3.new_workspace(1, 300, 300, 2)
    h3.h3attn_forward(d["q"], d["k"], d["v"], w.scale, view, ws)
    assert h3.h3attn_check_status(ws) == h3.OK
    compare_out(bits(view), oracle.attend_all(z, w.scale, EPOCH), "strided")
    assert (big[:, :, :, :64] == 7.0).all() and (big[:, :, :, 192:] == 7.0).all()


def test_repeated_launches_are_deterministic():
    """The fixed shape relaunched 1,000 times back to back gives the same output bytes
    every time (no hang, no race; the 1,000-launch check of "Phase 2B Aligned Numerical
    Prototype", Exactness)."""
    w = synth.WORKLOADS["fixed_q128_kv192"]
    x = synth.make_inputs(w)
    d = upload(x, w)
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    out = torch.empty(1, 128, 1, 128, dtype=torch.bfloat16, device="cuda")
    h3.h3attn_forward_ex(d["q"], d["k"], d["v"], w.scale, out, ws)
    first = out.clone()
    differs = torch.zeros((), dtype=torch.bool, device="cuda")
    for _ in range(1000):
        h3.h3attn_forward_ex(d["q"], d["k"], d["v"], w.scale, out, ws)
        differs |= (out.view(torch.int16) != first.view(torch.int16)).any()
    assert h3.h3attn_check_status(ws) == h3.OK
    assert not bool(differs)
    assert torch.equal(out.view(torch.int16), first.view(torch.int16))


def _field_sizes(B, Tq, Tkv, H):
    """Bytes each workspace field needs (the layout pads every field to 1024 bytes)."""
    Tqp, Tkp = -(-Tq // 128) * 128, -(-Tkv // 128) * 128
    nchunk = -(-Tkv // 64)
    BH = B * H
    return {"status": 12, "q8": 2 * BH * Tqp * 128, "k8": 2 * BH * Tkp * 128, "v8t": BH * 128 * Tkp,
            "sq": BH * Tqp // 32 * 4, "sk": BH * Tkp // 64 * 4, "km": BH * 128 * 4, "sv": BH * 128 * 4,
            "ksum": BH * nchunk * 128 * 8, "vmax": BH * nchunk * 128 * 4}


@pytest.mark.parametrize("B, Tq, Tkv, H", [(1, 300, 9453 // 3, 3), (2, 128, 192, 1)])
def test_workspace_guard_bands_stay_untouched(B, Tq, Tkv, H):
    """Canaries around the workspace and in the alignment gaps between its fields survive
    quantize and attend: no kernel writes outside the field it owns.  (Stands in for the
    memcheck runs of "Phase 2B Aligned Numerical Prototype", Synchronization And Safety,
    with compute-sanitizer closed on this pool.)"""
    w = synth.Workload("guard", B, Tq, Tkv, H, 128, "normal", 4242)
    x = synth.make_inputs(w)
    d = upload(x, w)
    n = h3.h3attn_workspace_bytes(B, Tq, Tkv, H)
    guard = 8192
    buf = torch.full((guard + n + guard,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = buf[guard:guard + n]
    out = torch.empty(B, Tq, H, 128, dtype=torch.bfloat16, device="cuda")
    h3.h3attn_forward_ex(d["q"], d["k"], d["v"], w.scale, out, ws)
    assert h3.h3attn_check_status(ws) == h3.OK
    host = buf.cpu().numpy()
    assert (host[:guard] == 0xA5).all() and (host[guard + n:] == 0xA5).all()
    off = h3.h3attn_workspace_layout(B, Tq, Tkv, H)
    need = _field_sizes(B, Tq, Tkv, H)
    names = h3.WS_FIELDS
    for a, b in zip(names[:-1], names[1:]):
        gap = host[guard + off[a] + need[a]: guard + off[b]]
        if a == "status":
            continue  # the status block's spare words belong to it
        assert (gap == 0xA5).all(), f"bytes after {a} were written"
    compare_out(bits(out), oracle.attend_all(oracle.quantize(x["q"], x["k"], x["v"]), w.scale, EPOCH), "guarded")


def test_full_size_soak_is_deterministic_and_never_times_out():
    """The H3-shaped call relaunched back to back: every launch must finish without a
    device-side timeout and produce the same bytes (a hand-off race shows up here as a
    stall, a timeout or a changed output; cf. the 1,000-launch soak of "Phase 2B
    Aligned Numerical Prototype", Exactness)."""
    w = synth.WORKLOADS["h3_t37810_h32"]
    x = synth.make_inputs(w)
    d = upload(x, w)
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    out = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device="cuda")
    h3.h3attn_quantize_qkv(d["q"], d["k"], d["v"], ws)
    h3.h3attn_attend(ws, w.B, w.Tq, w.Tkv, w.H, w.scale, out)
    assert h3.h3attn_check_status(ws) == h3.OK
    first = out.clone()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for _ in range(40):
        start.record()
        h3.h3attn_attend(ws, w.B, w.Tq, w.Tkv, w.H, w.scale, out)
        end.record()
        torch.cuda.synchronize()
        times.append(start.elapsed_time(end))
        assert torch.equal(out.view(torch.int16), first.view(torch.int16))
    assert h3.h3attn_check_status(ws) == h3.OK
    # no launch may stall: the slowest stays within 1.5x of the median
    times.sort()
    assert times[-1] < 1.5 * times[len(times) // 2], times


def test_trace_export_gives_the_same_output_and_a_timeline():
    """h3attn_debug_attend_trace runs the same kernel with a clock64 timeline in one CTA:
    the output bytes equal h3attn_attend's, and the traced CTA's per-tile events are
    ordered (scores ready -> probabilities computed -> handed over, tile after tile)."""
    w = synth.WORKLOADS["selfattn_h8_t4096"]
    x = synth.make_inputs(w)
    d = upload(x, w)
    ws, out, out4 = run_forward(w, d)
    traced = torch.empty_like(out4)
    ntq = -(-w.Tq // 128)
    ctas = ((ntq + 1) // 2) * w.H * w.B
    tr = h3.h3attn_debug_attend_trace(ws, w.B, w.Tq, w.Tkv, w.H, w.scale, traced, ctas // 2)
    assert h3.h3attn_check_status(ws) == h3.OK
    assert torch.equal(traced.view(torch.int16), out4.view(torch.int16))
    nkv = -(-w.Tkv // 128)
    for slot in (0, 1):
        s_ready, probs, p_done = (tr[n][slot].numpy().astype(np.int64) for n in ("s_ready", "probs", "p_done"))
        assert (s_ready > 0).all() and (probs > 0).all() and (p_done > 0).all()
        assert (s_ready < probs).all() and (probs < p_done).all()
        assert (np.diff(s_ready) > 0).all() and len(s_ready) == nkv


def test_forward_replays_from_a_cuda_graph():
    """The forward pass (four launches, no host synchronisation) can be captured once into a
    CUDA graph and replayed: every replay gives the bytes of a direct call."""
    w = synth.WORKLOADS["fixed_q128_kv192"]
    x = synth.make_inputs(w)
    d = upload(x, w)
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    direct = torch.empty(1, 128, 1, 128, dtype=torch.bfloat16, device="cuda")
    h3.h3attn_forward_ex(d["q"], d["k"], d["v"], w.scale, direct, ws)
    assert h3.h3attn_check_status(ws) == h3.OK
    out = torch.zeros_like(direct)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up on the capture stream
        h3.h3attn_forward_ex(d["q"], d["k"], d["v"], w.scale, out, ws)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        h3.h3attn_forward_ex(d["q"], d["k"], d["v"], w.scale, out, ws)
    for _ in range(50):
        out.zero_()
        g.replay()
        torch.cuda.current_stream().synchronize()
        assert torch.equal(out.view(torch.int16), direct.view(torch.int16))
    assert h3.h3attn_check_status(ws) == h3.OK


def test_concurrent_streams_with_separate_workspaces():
    """Two forward calls in flight at once on two streams, each with its own workspace,
    give the bytes of the same calls made one after the other (the library keeps no
    per-call global state)."""
    wa = synth.Workload("conc_a", 1, 700, 700, 4, 128, "normal", 8101)
    wb = synth.Workload("conc_b", 2, 333, 900, 3, 128, "k_offset", 8102)
    runs = []
    for w in (wa, wb):
        x = synth.make_inputs(w)
        d = upload(x, w)
        ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
        ref = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device="cuda")
        h3.h3attn_forward_ex(d["q"], d["k"], d["v"], w.scale, ref, ws)
        assert h3.h3attn_check_status(ws) == h3.OK
        runs.append((w, d, h3.new_workspace(w.B, w.Tq, w.Tkv, w.H), ref))
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [torch.zeros_like(r[3]) for r in runs]
    torch.cuda.synchronize()
    for _ in range(5):
        for (w, d, ws, _), s, o in zip(runs, streams, outs):
            h3.h3attn_forward_ex(d["q"], d["k"], d["v"], w.scale, o, ws, stream=s)
    torch.cuda.synchronize()
    for (w, d, ws, ref), s, o in zip(runs, streams, outs):
        assert h3.h3attn_check_status(ws, s) == h3.OK
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16)), w.name


def test_random_shapes_against_the_oracle():
    """A seeded sweep of shapes (batch, ragged lengths, Tq != Tkv, heads, packed or
    separate layouts): integer stages bit-exact, outputs within tolerance."""
    rng = np.random.default_rng(20261202)
    for case in range(8):
        B = int(rng.integers(1, 3))
        Tq = int(rng.integers(1, 700))
        Tkv = Tq if case % 2 == 0 else int(rng.integers(1, 900))
        H = int(rng.integers(1, 5))
        packed = case % 2 == 0
        recipe = ("normal", "k_offset", "rmsnorm")[case % 3]
        w = synth.Workload(f"rand_{case}", B, Tq, Tkv, H, 128, recipe, 9000 + case, packed=packed)
        x = synth.make_inputs(w)
        z = oracle.quantize(x["q"], x["k"], x["v"])
        d = upload(x, w)
        ws, out, out4 = run_forward(w, d)
        check_quantized(ws, z, w)
        compare_out(bits(out4), oracle.attend_all(z, w.scale, EPOCH), w.name)


def test_concurrent_host_threads():
    """Four host threads call the library at once (ctypes releases the GIL), each on its
    own stream and workspace; every output equals the single-threaded result."""
    import threading
    w = synth.Workload("threads", 1, 600, 600, 2, 128, "rmsnorm", 8201)
    x = synth.make_inputs(w)
    d = upload(x, w)
    ws0 = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    ref = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device="cuda")
    h3.h3attn_forward(d["q"], d["k"], d["v"], w.scale, ref, ws0)
    assert h3.h3attn_check_status(ws0) == h3.OK
    n = 4
    streams = [torch.cuda.Stream() for _ in range(n)]
    wss = [h3.new_workspace(w.B, w.Tq, w.Tkv, w.H) for _ in range(n)]
    outs = [torch.zeros_like(ref) for _ in range(n)]
    errors = []
    torch.cuda.synchronize()

    def worker(i):
        try:
            torch.cuda.set_device(0)
            for _ in range(10):
                h3.h3attn_forward(d["q"], d["k"], d["v"], w.scale, outs[i], wss[i], stream=streams[i])
            if h3.h3attn_check_status(wss[i], streams[i]) != h3.OK:
                errors.append(f"thread {i}: device status")
        except Exception as e:  # reported below, in the test's own thread
            errors.append(f"thread {i}: {e!r}")

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(n)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    torch.cuda.synchronize()
    for o in outs:
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))

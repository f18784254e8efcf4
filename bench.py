"""Benchmark: quantized attention effective TOPS and ms per call on B200.

One step = one ``h3attn_forward`` call (K smoothing + Q/K/V quantization +
the fused attention mainloop) over the H3-shaped packed video+text sequence
(B=1, T=37,810, H=32, D=128).  Effective TOPS = 4*B*Tq*Tkv*H*D / time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Under torchrun (N > 1) every rank runs its own copy of the workload on its own
GPU (independent problems, weak scaling, no data-path collective); timing is
the max over ranks.  ``--impl reference`` times the CPU oracle on the host
cores on a bounded sample of the same workload (rank 0 only).

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "quantized attention effective TOPS and ms/call at T=37,810, H=32, D=128 (1xB200)"


def metric_of(w) -> str:
    """The headline metric string; other workloads name their own sizes."""
    if w.name == DEFAULT_WORKLOAD:
        return METRIC
    return "quantized attention%s effective TOPS and ms/call at Tq=%s, Tkv=%s, B=%d, H=%d, D=%d (1xB200)" % (
        " with Q/K RMSNorm + RoPE" if w.norm_rope else "", format(w.Tq, ","), format(w.Tkv, ","), w.B, w.H, w.D)
UNIT = "TOPS"
DEFAULT_WORKLOAD = "h3_t37810_h32"
KERNEL_SOURCES = ["quantized_attention_video_b200/csrc/attention.cu", "quantized_attention_video_b200/csrc/sm100_ptx.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample-rows", type=int, default=0,
                    help="query rows of head 0 timed on the CPU oracle (0 = all Tq rows of that head)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-heads-per-group", type=int, default=2,
                    help="head group of the pipelined host-buffer forward pass (h3attn_forward_host)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--heads", type=int, default=0,
                    help="override H (a smaller case of the same kernel for profiler captures)")
    ap.add_argument("--latency", action="store_true",
                    help="per-call latency of the fixed 128 x 192 shape by the pages' method (samples of 20 "
                         "back-to-back calls, p50 and CV), forward and attend-only samples alternated")
    ap.add_argument("--samples", type=int, default=500)
    ap.add_argument("--ulysses", action="store_true",
                    help="one sequence of the workload spread over the GPUs by tokens: head-sharding all-to-alls "
                         "around the attention of H/N heads per GPU (strong scaling)")
    return ap.parse_args()


def dist_env():
    # NCCL prints its version banner on stdout unless told otherwise; the bench's stdout is
    # its one JSON line
    os.environ.setdefault("NCCL_DEBUG", "WARN")
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def config_of(w: synth.Workload, world: int) -> dict:
    return {"workload": w.name, "B": w.B, "Tq": w.Tq, "Tkv": w.Tkv, "H": w.H, "D": w.D,
            "layout": "packed [B,T,3,H,D] in, [B,T,H*D] out" if w.packed else "separate [B,T,H,D] in and out",
            "inputs": f"seeded synthetic ({w.recipe}), seed {w.seed}" + (
                "; Q/K RMSNorm + RoPE (gamma ~ N(1, 0.1), eps 1e-6, 3-axis video rotary tables, last 100 tokens "
                "unrotated) fused into the preparation" if w.norm_rope else ""),
            "l2": "inputs + workspace > 126 MB L2; no flush between steps",
            "parallelism": f"independent replica per GPU x{world}" if world > 1 else "single GPU"}


# ------------------------------------------------------------ CPU oracle ----
def cpu_oracle_sample(w: synth.Workload, rows_per_head: int, x=None):
    """Time the oracle on a bounded sample: quantize of one head plus attention of
    `rows_per_head` query rows of that head.  Returns (TOPS, seconds, threads, text)."""
    import oracle
    oracle.build()
    if x is None:
        x = synth.make_inputs(w)
    q, k, v = (x[n][:, :, :1] for n in ("q", "k", "v"))
    threads = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    if w.norm_rope:
        z = oracle.quantize_norm_rope(q, k, v, synth.norm_rope_params(w))
    else:
        z = oracle.quantize(q, k, v)
    t_quant = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    if rows_per_head <= 0 or rows_per_head >= w.Tq:
        rows_per_head = w.Tq
        picked = np.arange(w.Tq)
    else:
        picked = np.sort(rng.choice(w.Tq, rows_per_head, replace=False))
    rows = np.stack([np.zeros(rows_per_head, int), np.zeros(rows_per_head, int), picked], axis=1)
    t0 = time.perf_counter()
    oracle.attend_rows(z, w.scale, 128, rows)
    t_rows = time.perf_counter() - t0
    # the quantize pass is shared by all Tq rows of the head; charge its share
    secs = t_rows + t_quant * rows_per_head / w.Tq
    ops = 4.0 * rows_per_head * w.Tkv * w.D
    what = "all" if rows_per_head == w.Tq else f"{rows_per_head} random"
    text = (f"{w.name}: quantize of 1 of {w.B * w.H} heads ({t_quant:.2f} s, charged pro rata) + attention "
            f"of {what} query rows of it ({t_rows:.2f} s) on {threads} threads")
    return ops / secs / 1e12, secs, threads, text


def run_reference(args, w):
    rank, _, world = dist_env()
    if rank != 0:
        return
    K = max(1, args.steps)
    vals = []
    x = synth.make_inputs(w)
    info = None
    # each step: one head's quantize (charged pro rata) + 2,048 query rows, about a second
    rows = args.cpu_sample_rows if args.cpu_sample_rows > 0 else 2048
    if args.warmup > 0:
        cpu_oracle_sample(w, 64, x)
    for _ in range(K):
        tops, secs, threads, text = cpu_oracle_sample(w, rows, x)
        vals.append(tops)
        info = (threads, text)
    value = statistics.median(vals)
    ms = 4.0 * w.B * w.Tq * w.Tkv * w.H * w.D / (value * 1e12) * 1e3
    line = {"impl": "reference", "metric": metric_of(w), "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8/e4m3 (fp32 softmax)", "data": "synthetic",
            "config": config_of(w, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": info[0], "kind": "oracle", "sample": info[1]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "note": "CPU oracle on host cores; ms_per_step extrapolates the sampled rate to the whole call"}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ clocks ----
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"h3attn_clocks_{os.getpid()}_{index}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [s.strip() for s in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax = float(p[2])
            except ValueError:
                continue
            for n, val in zip(names, p[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def traffic_record(w):
    """DRAM bytes per attention launch from the committed ncu summary, if it was
    taken on the current kernel source and this workload (else None)."""
    path = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path))
    if rec.get("workload") != w.name:
        return None
    h = hashlib.sha256()
    for src in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, src), "rb").read())
    if rec.get("kernel_sha256") != h.hexdigest():
        return None
    return rec


def launches_per_step(w) -> int:
    """Kernels one forward launches: the preparation (one kernel for sequences of at most 4
    slabs of 128 tokens, else statistics + ordered reduction + quantize, plus the Q transform
    with the norm + RoPE) and the attention."""
    slabs = max(-(-w.Tq // 128), -(-w.Tkv // 128))
    prep = 1 if slabs <= 4 else 3 + (1 if w.norm_rope else 0)
    return prep + 1


def max_over_ranks(dist, val: float, device) -> float:
    """The slowest rank's value (all ranks take part; dist None = single process)."""
    if dist is None:
        return val
    import torch
    t = torch.tensor([val], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(ops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput of independent replicas (weak scaling): every rank does
    ops_per_rank per step and the job is as slow as its slowest rank.  TOPS."""
    return world * ops_per_rank / (ms_per_step * 1e-3) / 1e12


# --------------------------------------------------------------- GPU arm ----
def run_ours(args, w):
    import torch
    import quantized_attention_video_b200 as h3
    from quantized_attention_video_b200 import build as h3build

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    if rank == 0 or not os.path.exists(h3build.SO):
        h3build.build()
    if dist is not None:
        dist.barrier()
    h3.lib()

    x = synth.make_inputs(w)
    ops = w.ops
    dev = torch.device("cuda", local)

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)

    if w.packed:
        buf = to_dev(x["packed"])
        q, k, v = buf[:, :, 0], buf[:, :, 1], buf[:, :, 2]
        out_flat = torch.empty(w.B, w.Tq, w.H * w.D, dtype=torch.bfloat16, device=dev)
        out = out_flat.view(w.B, w.Tq, w.H, w.D)
    else:
        q, k, v = (to_dev(x[n]) for n in ("q", "k", "v"))
        out = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device=dev)
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H, device=dev)
    stream = torch.cuda.current_stream(dev)
    nr = None
    if w.norm_rope:
        nr_host = synth.norm_rope_params(w)
        nr = {n: torch.from_numpy(np.ascontiguousarray(nr_host[n])).to(dev) for n in h3.NORM_ROPE_FIELDS}
        nr["eps"] = nr_host["eps"]

    def prep():
        if nr is None:
            h3.h3attn_quantize_qkv(q, k, v, ws, stream)
        else:
            h3.h3attn_quantize_qkv_norm_rope(q, k, v, nr, ws, stream)

    def step():
        prep()
        h3.h3attn_attend(ws, w.B, w.Tq, w.Tkv, w.H, w.scale, out, stream)

    for _ in range(max(3, args.warmup)):
        step()
    if h3.h3attn_check_status(ws, stream) != h3.OK:
        raise RuntimeError("device status not OK after warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(K):
        ev[i][0].record(stream)
        prep()
        ev[i][1].record(stream)
        h3.h3attn_attend(ws, w.B, w.Tq, w.Tkv, w.H, w.scale, out, stream)
        ev[i][2].record(stream)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    total_ms = ev[0][0].elapsed_time(ev[K - 1][2])
    quant_ms = [e[0].elapsed_time(e[1]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    if h3.h3attn_check_status(ws, stream) != h3.OK:
        raise RuntimeError("device status not OK after the timed steps")

    total_ms = max_over_ranks(dist, total_ms, dev)
    ms_step = total_ms / K
    value = job_rate(ops, world, ms_step)
    attn_avg = max_over_ranks(dist, statistics.mean(attn_ms), dev)
    quant_avg = max_over_ranks(dist, statistics.mean(quant_ms), dev)

    # ------------------------------------------ fused vs separate norm + RoPE
    norm_rope = None
    if nr is not None:
        # the same preparation as a separate norm + RoPE pass over Q and K (written to
        # scratch tensors) followed by the plain preparation
        qn, kn = torch.empty_like(q), torch.empty_like(k)
        ws2 = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H, device=dev)

        def separate():
            h3.h3attn_norm_rope(q, nr["gamma_q"], nr["cos_q"], nr["sin_q"], nr["eps"], qn, stream)
            h3.h3attn_norm_rope(k, nr["gamma_k"], nr["cos_k"], nr["sin_k"], nr["eps"], kn, stream)

        for _ in range(3):
            separate()
            h3.h3attn_quantize_qkv(qn, kn, v, ws2, stream)
        Kn = max(5, K // 2)
        evn = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(Kn)]
        torch.cuda.synchronize(dev)
        for i in range(Kn):
            evn[i][0].record(stream)
            separate()
            evn[i][1].record(stream)
            h3.h3attn_quantize_qkv(qn, kn, v, ws2, stream)
            evn[i][2].record(stream)
        torch.cuda.synchronize(dev)
        sep_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evn)
        plain_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evn)
        norm_rope = {"fused_prep_ms": max_over_ranks(dist, statistics.mean(quant_ms), dev),
                     "separate_pass_ms": max_over_ranks(dist, sep_ms, dev),
                     "plain_prep_ms": max_over_ranks(dist, plain_ms, dev),
                     "separate_pass_gbs": 4.0 * (w.Tq + w.Tkv) * w.B * w.H * w.D / (sep_ms * 1e-3) / 1e9,
                     "note": "fused = h3attn_quantize_qkv_norm_rope; separate = h3attn_norm_rope on Q and K "
                             "(read + write 2 B each, plus 2 x 256 B of tables per token) then h3attn_quantize_qkv"}
        if h3.h3attn_check_status(ws2, stream) != h3.OK:
            raise RuntimeError("device status not OK in the separate-pass timing")

    # ------------------------------------------------ end to end (host buffers)
    e2e = None
    if not args.no_e2e and nr is None:
        # pinned host inputs and output; the library uploads, computes and downloads
        # head groups on overlapping streams (h3attn_forward_host)
        if w.packed:
            h_in = [torch.from_numpy(x["packed"].view(np.int16)).view(torch.bfloat16).pin_memory()]
            hq, hk, hv = (h_in[0][:, :, i] for i in range(3))
        else:
            h_in = [torch.from_numpy(np.ascontiguousarray(x[n]).view(np.int16)).view(torch.bfloat16).pin_memory()
                    for n in ("q", "k", "v")]
            hq, hk, hv = h_in
        h_out = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in h_in)
        d2h = h_out.numel() * h_out.element_size()
        g = max(1, min(args.e2e_heads_per_group, w.H))
        hbuf = h3.new_host_buffer(w.B, w.Tq, w.Tkv, w.H, g)

        def e2e_step():
            h3.h3attn_forward_host(hq, hk, hv, w.scale, h_out, hbuf, g, stream)

        Ke = max(3, K // 4)
        for _ in range(2):
            e2e_step()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(Ke):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(dist, e0.elapsed_time(e1) / Ke, dev)
        e2e = {"value": job_rate(ops, world, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms, "steps": Ke,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "path": "pinned host Q/K/V -> h3attn_forward_host (upload, forward and download of head groups of %d "
                       "on overlapping streams) -> pinned host out" % g}
        if h3.h3attn_forward_host_check_status(hbuf, w.B, w.Tq, w.Tkv, w.H, g, stream) != h3.OK:
            raise RuntimeError("device-side failure in the end-to-end pass")

    peaks = {}
    pk_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk_path):
        peaks = json.load(open(pk_path))
    # The attention kernel runs inside a step of tens of milliseconds, not a seconds-long
    # loop, so the burst GEMM rate is its peak; the sustained (power-capped) rate is
    # reported beside it for reference.  8-bit dense = 2 x bf16 dense (nominal ratio).
    if "bf16_tflops" in peaks:
        peak = 2.0 * peaks["bf16_tflops"]
        peak_note = "of measured: 2 x bf16_tflops (burst; nominal 8-bit/bf16 ratio 2)"
    else:
        peak = 2.0 * 1590.0
        peak_note = "of fallback: 2 x 1.59 PFLOP/s burst bf16"
    achieved = ops / (attn_avg * 1e-3) / 1e12
    tr = traffic_record(w)
    bthd = w.B * w.H * w.D
    # the method's bytes: stats reads K, V (4 B per key); quantize reads Q (2 B), K, V (4 B)
    # and writes the INT8 Q and K words and the E4M3 V words (1 B each): 13 B per token at
    # Tq = Tkv.  The Q/K words are stored as BF16 values (2 B each): one extra byte per
    # word, reported on its own.
    quant_bytes = (3 * w.Tq + 10 * w.Tkv) * bthd
    word_overhead = (w.Tq + w.Tkv) * bthd
    roofline = {"bound": "tensor", "kernel": "attn_sm100_kernel", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "peak_source": peak_note,
                "algorithmic_ops_per_launch": ops,
                "traffic": None if tr is None else tr["dram_bytes_per_launch_full"],
                "quantize_ms": quant_avg, "attention_ms": attn_avg,
                "quantize_algorithmic_bytes": quant_bytes,
                "quantize_gbs": quant_bytes / (quant_avg * 1e-3) / 1e9,
                "quantize_word_overhead_bytes": word_overhead}
    if "bf16_tflops_sustained" in peaks:
        roofline["peak_sustained"] = 2.0 * peaks["bf16_tflops_sustained"]
        roofline["frac_of_sustained"] = achieved / roofline["peak_sustained"]
    if "hbm_gbs" in peaks:
        # the preparation kernels are HBM-bound: their algorithmic bytes against the measured copy rate
        roofline["quantize_frac_of_hbm"] = roofline["quantize_gbs"] / peaks["hbm_gbs"]
        roofline["hbm_peak_gbs"] = peaks["hbm_gbs"]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tops, secs, threads, text = cpu_oracle_sample(w, args.cpu_sample_rows, x)
        cpu = {"value": tops, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": text}

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": metric_of(w), "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "i8/e4m3 (fp32 softmax)", "data": "synthetic", "config": config_of(w, world),
            "clocks": clk, "gpu_launches": launches_per_step(w) * K, "roofline": roofline, "e2e": e2e,
            "cpu_baseline": cpu}
    if norm_rope is not None:
        line["norm_rope"] = norm_rope
        line["e2e_note"] = "the host-buffer pipeline has no norm + RoPE variant; e2e is measured on the plain workloads"
    print(json.dumps(line), flush=True)


# --------------------------------------------------------- Ulysses mode ----
def run_ulysses(args, w):
    """One sequence of the workload spread over the ranks by tokens (strong scaling: the
    whole job is one problem).  Each step: the token-to-head all-to-all of Q, K and V, the
    library forward pass on this rank's H/N heads, the head-to-token all-to-all of the
    output.  Inputs resident on the GPUs; CUDA events around each part, max over ranks."""
    import dataclasses
    import datetime
    import socket

    import torch
    import torch.distributed as dist
    import quantized_attention_video_b200 as h3
    from quantized_attention_video_b200 import build as h3build
    from quantized_attention_video_b200 import ulysses

    if w.packed or w.norm_rope or w.Tq != w.Tkv:
        raise SystemExit("--ulysses takes a self-attention workload in the separate layout")
    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world == 1 and "MASTER_ADDR" not in os.environ:
        with socket.socket() as sck:
            sck.bind(("127.0.0.1", 0))
            port = sck.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=120), device_id=dev)
    else:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if w.H % world:
        raise SystemExit(f"{w.H} heads do not split over {world} GPUs")
    if rank == 0 or not os.path.exists(h3build.SO):
        h3build.build()
    dist.barrier()
    h3.lib()

    x = synth.make_inputs(w)
    counts = ulysses.token_counts(w.Tq, world)
    off = sum(counts[:rank])
    q, k, v = (torch.from_numpy(np.ascontiguousarray(x[n][:, off:off + counts[rank]]).view(np.int16)).to(dev)
               .view(torch.bfloat16) for n in ("q", "k", "v"))
    del x
    hn = w.H // world
    ws = h3.new_workspace(w.B, w.Tq, w.Tq, hn, device=dev)
    oh = torch.empty(w.B, w.Tq, hn, w.D, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        qh, kh, vh = ulysses.seq_to_head([q, k, v], w.Tq)
        if ev:
            ev[1].record(stream)
        h3.h3attn_forward_ex(qh, kh, vh, w.scale, oh, ws, stream)
        if ev:
            ev[2].record(stream)
        o = ulysses.head_to_seq(oh, w.Tq)
        if ev:
            ev[3].record(stream)
        return o

    for _ in range(max(3, args.warmup)):
        step()
    if h3.h3attn_check_status(ws, stream) != h3.OK:
        raise RuntimeError("device status not OK after warm-up")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(K):
        step(ev[i])
    torch.cuda.synchronize(dev)
    dist.barrier()
    clk = clocks.stop()
    if h3.h3attn_check_status(ws, stream) != h3.OK:
        raise RuntimeError("device status not OK after the timed steps")
    total_ms = max_over_ranks(dist, ev[0][0].elapsed_time(ev[K - 1][3]), dev)
    to_head = max_over_ranks(dist, statistics.mean(e[0].elapsed_time(e[1]) for e in ev), dev)
    compute = max_over_ranks(dist, statistics.mean(e[1].elapsed_time(e[2]) for e in ev), dev)
    to_seq = max_over_ranks(dist, statistics.mean(e[2].elapsed_time(e[3]) for e in ev), dev)
    dist.barrier()
    dist.destroy_process_group()
    if rank != 0:
        return
    ms_step = total_ms / K
    shard_bytes = 3 * w.B * counts[0] * w.H * w.D * 2  # Q, K and V of the largest token shard
    cfg = config_of(w, world)
    cfg["parallelism"] = (f"Ulysses over {world} GPU(s): token shards of {counts[-1]}-{counts[0]} tokens, "
                          f"{hn} heads per GPU, NCCL all-to-all before and after")
    line = {"metric": metric_of(w).replace("(1xB200)", f"({world}xB200, one sequence)"),
            "value": w.ops / (ms_step * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "i8/e4m3 (fp32 softmax)", "data": "synthetic", "config": cfg,
            "clocks": clk, "gpu_launches": launches_per_step(dataclasses.replace(w, H=hn)) * K,
            "ulysses": {"seq_to_head_ms": to_head, "forward_ms": compute, "head_to_seq_ms": to_seq,
                        "bytes_per_rank_to_head": shard_bytes, "bytes_per_rank_to_seq": shard_bytes // 3},
            "e2e": None, "cpu_baseline": None}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------- latency mode ----
def run_latency(args):
    """Per-call latency at the fixed shape (B1 H1 Tq128 Tkv192 D128), measured the way the
    pages measure it ("Phase 2B Aligned Numerical Prototype", the batched p50 over samples
    of 20 back-to-back launches, with CV): each sample times 20 calls with CUDA events.
    Forward and attend-only samples alternate in the same process so that clock changes
    fall on both; a third series replays one CUDA graph of 20 forward calls."""
    import torch
    import quantized_attention_video_b200 as h3
    from quantized_attention_video_b200 import build as h3build

    h3build.build()
    h3.lib()
    w = synth.WORKLOADS["fixed_q128_kv192"]
    x = synth.make_inputs(w)

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)

    q, k, v = dev(x["q"]), dev(x["k"]), dev(x["v"])
    out = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device="cuda")
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    per = 20

    def forward():
        h3.h3attn_forward_ex(q, k, v, w.scale, out, ws)

    def attend():
        h3.h3attn_attend(ws, w.B, w.Tq, w.Tkv, w.H, w.scale, out)

    for _ in range(max(50, args.warmup)):
        forward()
    if h3.h3attn_check_status(ws) != h3.OK:
        raise RuntimeError("device status not OK after warm-up")
    cur = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    side.wait_stream(cur)
    with torch.cuda.stream(side):
        forward()
    cur.wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(per):
            forward()

    def sample(run) -> float:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) / per

    series = {"forward": [], "attend": [], "graph": []}
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    for _ in range(args.samples):
        series["forward"].append(sample(lambda: [forward() for _ in range(per)]))
        series["attend"].append(sample(lambda: [attend() for _ in range(per)]))
        series["graph"].append(sample(graph.replay))
    clk = clocks.stop()
    if h3.h3attn_check_status(ws) != h3.OK:
        raise RuntimeError("device status not OK after the samples")

    def summary(vals):
        return {"p50_ms": statistics.median(vals), "cv": statistics.pstdev(vals) / statistics.mean(vals)}

    fwd = summary(series["forward"])
    line = {"metric": "per-call latency, p50 of samples of 20 back-to-back calls, at Tq=128, Tkv=192, B=1, H=1, "
                      "D=128 (1xB200)",
            "value": fwd["p50_ms"], "unit": "ms", "higher_is_better": False, "cv": fwd["cv"],
            "samples": args.samples, "calls_per_sample": per,
            "attend_only": summary(series["attend"]), "forward_graph_of_20": summary(series["graph"]),
            "data": "synthetic", "config": dict(config_of(w, 1), l2="the shape's 0.2 MB stays in L2; no flush, as "
                                                                   "in the pages' method"), "clocks": clk,
            "note": "forward = h3attn_forward_ex (one preparation launch + the attention launch); samples of "
                    "the three series interleaved"}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.latency:
        run_latency(args)
        return
    w = synth.WORKLOADS[args.workload]
    if args.heads:
        import dataclasses
        w = dataclasses.replace(w, name=f"{w.name}_h{args.heads}", H=args.heads)
    if args.impl == "reference":
        run_reference(args, w)
    elif args.ulysses:
        run_ulysses(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()

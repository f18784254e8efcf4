"""The Ulysses exchange (quantized_attention_video_b200/ulysses.py) on gloo ranks (CPU).

One sequence is spread over two (or three) ranks by tokens (ragged: 301 tokens give
shards of 151 and 150; 100 tokens over three ranks 34, 33 and 33).  seq_to_head must hand every rank all tokens of its H/2 heads, head_to_seq
must invert it, and the composition with a per-head attention must give, on each
rank's tokens, the bytes that one process computing every head produces.  The
attention used here is the oracle's (the GPU library has no CPU path), so the
comparison is with the oracle run on the whole problem in this process.
"""
import datetime
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth

CASES = {  # name: (B, T, H, seed)
    "ulysses_b1_t301_h4": (1, 301, 4, 5101),
    "ulysses_b2_t200_h2": (2, 200, 2, 5102),
}


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload(name):
    B, T, H, seed = CASES[name]
    return synth.Workload(name, B, T, T, H, 128, "rmsnorm", seed)


def _oracle_attention(q, k, v, scale):
    """Per-head attention of [B, T, Hn, D] BF16 bit patterns (torch int16) by the oracle."""
    qa, ka, va = (t.contiguous().numpy().view(np.uint16) for t in (q, k, v))
    z = oracle.quantize(qa, ka, va)
    return torch.from_numpy(oracle.attend_all(z, scale, 128).view(np.int16))


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        from quantized_attention_video_b200 import ulysses
        for name in CASES:
            w = _workload(name)
            x = synth.make_inputs(w)
            counts = ulysses.token_counts(w.Tq, world)
            off = sum(counts[:rank])
            q, k, v = (torch.from_numpy(np.ascontiguousarray(x[n][:, off:off + counts[rank]]).view(np.int16))
                       for n in "qkv")
            qh, kh, vh = ulysses.seq_to_head([q, k, v], w.Tq)
            np.save(os.path.join(out_dir, f"{name}_qh{rank}.npy"), qh.numpy())
            np.save(os.path.join(out_dir, f"{name}_vh{rank}.npy"), vh.numpy())
            back = ulysses.head_to_seq(kh, w.Tq)
            np.save(os.path.join(out_dir, f"{name}_kback{rank}.npy"), back.numpy())
            out = ulysses.ulysses_attention(q, k, v, w.Tq, w.scale, attend=_oracle_attention)
            np.save(os.path.join(out_dir, f"{name}_out{rank}.npy"), out.numpy())
        # refused shapes: a head count the ranks cannot split, a shard of the wrong length
        errors = []
        for bad in ("heads", "tokens"):
            try:
                if bad == "heads":
                    t = torch.zeros(1, ulysses.token_counts(10, world)[rank], 3, 128, dtype=torch.int16)
                    ulysses.seq_to_head([t], 10)
                else:
                    t = torch.zeros(1, 7, 2, 128, dtype=torch.int16)
                    ulysses.seq_to_head([t], 10)
                errors.append(f"{bad}: accepted")
            except ValueError:
                errors.append(f"{bad}: refused")
        with open(os.path.join(out_dir, f"errors{rank}.txt"), "w") as f:
            f.write("\n".join(errors))
    finally:
        dist.destroy_process_group()


def test_two_ranks_give_the_single_process_bytes(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for name in CASES:
        w = _workload(name)
        x = synth.make_inputs(w)
        Hn = w.H // world
        counts = [w.Tq // world + (1 if r < w.Tq % world else 0) for r in range(world)]
        load = lambda what, r: np.load(tmp_path / f"{name}_{what}{r}.npy").view(np.uint16)
        for r in range(world):
            # every token of rank r's heads, in token order
            assert np.array_equal(load("qh", r), x["q"][:, :, r * Hn:(r + 1) * Hn]), (name, r)
            assert np.array_equal(load("vh", r), x["v"][:, :, r * Hn:(r + 1) * Hn]), (name, r)
            # the round trip returns each rank's own shard
            off = sum(counts[:r])
            assert np.array_equal(load("kback", r), x["k"][:, off:off + counts[r]]), (name, r)
        ref = oracle.attend_all(oracle.quantize(x["q"], x["k"], x["v"]), w.scale, 128)
        got = np.concatenate([load("out", r) for r in range(world)], axis=1)
        assert got.shape == ref.shape
        assert np.array_equal(got, ref), name
    for r in range(world):
        assert open(tmp_path / f"errors{r}.txt").read().split("\n") == ["heads: refused", "tokens: refused"]


def _rank_three(rank: int, world: int, port: int, out_dir: str):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        from quantized_attention_video_b200 import ulysses
        w = synth.Workload("ulysses_b1_t100_h6", 1, 100, 100, 6, 128, "k_offset", 5103)
        x = synth.make_inputs(w)
        counts = ulysses.token_counts(w.Tq, world)
        off = sum(counts[:rank])
        q, k, v = (torch.from_numpy(np.ascontiguousarray(x[n][:, off:off + counts[rank]]).view(np.int16))
                   for n in "qkv")
        out = ulysses.ulysses_attention(q, k, v, w.Tq, w.scale, attend=_oracle_attention)
        np.save(os.path.join(out_dir, f"three_out{rank}.npy"), out.numpy())
    finally:
        dist.destroy_process_group()


def test_three_ranks_with_a_ragged_split(tmp_path):
    """100 tokens over three ranks (34, 33, 33), 6 heads (2 per rank)."""
    world = 3
    mp.start_processes(_rank_three, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    w = synth.Workload("ulysses_b1_t100_h6", 1, 100, 100, 6, 128, "k_offset", 5103)
    x = synth.make_inputs(w)
    ref = oracle.attend_all(oracle.quantize(x["q"], x["k"], x["v"]), w.scale, 128)
    got = np.concatenate([np.load(tmp_path / f"three_out{r}.npy").view(np.uint16) for r in range(world)], axis=1)
    assert [np.load(tmp_path / f"three_out{r}.npy").shape[1] for r in range(world)] == [34, 33, 33]
    assert np.array_equal(got, ref)


def test_token_counts_split_raggedly():
    from quantized_attention_video_b200.ulysses import token_counts
    assert token_counts(301, 2) == [151, 150]
    assert token_counts(37810, 8) == [4727, 4727, 4726, 4726, 4726, 4726, 4726, 4726]
    assert sum(token_counts(74000, 3)) == 74000

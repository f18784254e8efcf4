"""The N>1 path of bench.py without a GPU: two gloo ranks on 127.0.0.1.

bench.py runs one independent replica of the workload per GPU (weak scaling, no
data-path collective; the (b, h) problems are independent).  What crosses ranks is
host-side: every rank takes part in the same barriers and reductions, the job is as
slow as its slowest rank, the whole-job rate counts every rank's work, and rank 0
alone prints.  These tests check that logic with CPU tensors."""
import datetime
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, ops: float, out_dir: str):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        b = _bench()
        local_ms = 10.0 + rank  # rank r took 10 + r ms per step
        dist.barrier()
        ms = b.max_over_ranks(dist, local_ms, "cpu")
        rate = b.job_rate(ops, world, ms)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{ms!r} {rate!r}\n")
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_rank_and_the_job_rate(tmp_path):
    ops, world = 23.4225e12, 2
    mp.start_processes(_rank_main, args=(world, _free_port(), ops, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = [open(tmp_path / f"rank{r}.txt").read().split() for r in range(world)]
    for ms, rate in got:
        assert float(ms) == 11.0  # the slower rank
        assert float(rate) == pytest.approx(world * ops / 11e-3 / 1e12, rel=1e-12)


def test_single_process_helpers():
    b = _bench()
    assert b.max_over_ranks(None, 7.5, "cpu") == 7.5
    assert b.job_rate(1e12, 1, 1000.0) == pytest.approx(1.0)
    assert b.job_rate(1e12, 8, 1000.0) == pytest.approx(8.0)  # weak scaling: 8 replicas, same time


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    b = _bench()
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert b.run_reference(None, None) is None  # returns before touching its arguments
    assert capsys.readouterr().out == ""


def test_replica_config_names_the_parallelism():
    import synth
    b = _bench()
    w = synth.WORKLOADS["h3_t37810_h32"]
    assert b.config_of(w, 1)["parallelism"] == "single GPU"
    assert "x4" in b.config_of(w, 4)["parallelism"]

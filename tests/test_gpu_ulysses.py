"""The Ulysses path (quantized_attention_video_b200/ulysses.py) on the GPU through NCCL.

A run gets one GPU, so the process group has one rank: the all-to-alls move every
byte to the same rank, which still exercises the NCCL calls, the byte views and the
library attention on the exchanged head shards.  The output must be the bytes of the
library's forward pass on the unsharded inputs.  The exchange logic for two ranks is
tested on CPU (tests/test_ulysses.py)."""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import synth
import quantized_attention_video_b200 as h3

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_attention_video_b200 import build
    build.build()
    h3.lib()


def test_single_rank_exchange_gives_the_library_bytes():
    from quantized_attention_video_b200 import ulysses
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=120))
    try:
        for name in ("selfattn_h8_t4096", "ragged_h16_t9453"):
            w = synth.WORKLOADS[name]
            x = synth.make_inputs(w)
            q, k, v = (torch.from_numpy(np.ascontiguousarray(x[n]).view(np.int16)).cuda().view(torch.bfloat16)
                       for n in "qkv")
            out = ulysses.ulysses_attention(q, k, v, w.Tq, w.scale)
            ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
            ref = torch.empty_like(q)
            h3.h3attn_forward_ex(q, k, v, w.scale, ref, ws)
            assert h3.h3attn_check_status(ws) == h3.OK
            torch.cuda.synchronize()
            assert out.shape == ref.shape
            assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), name
    finally:
        dist.destroy_process_group()

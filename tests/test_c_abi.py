"""The C ABI used from plain C: tests/c_abi_forward.c includes only include/h3attn.h and
the CUDA runtime, allocates its own device buffers and calls h3attn_forward_ex.

CPU: the program compiles and links against libh3attn.so (every function it calls
resolves).  GPU: it runs the fixed 128 x 192 problem and writes the same output bytes as
the Python binding's call on the same inputs (one library, two callers).
"""
import os
import shutil
import struct
import subprocess

import numpy as np
import pytest

import synth
import quantized_attention_video_b200 as h3

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi_forward.c")
OUT_DIR = os.path.join(ROOT, "_build")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def build_program() -> str:
    from quantized_attention_video_b200 import build
    build.build()
    os.makedirs(OUT_DIR, exist_ok=True)
    exe = os.path.join(OUT_DIR, "c_abi_forward")
    libdir = os.path.dirname(h3.LIB_PATH)
    cc = shutil.which("gcc") or "cc"
    subprocess.check_call([cc, "-std=c11", "-O2", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(CUDA, "include"), SRC, "-o", exe, "-L", libdir, "-lh3attn",
                           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{libdir}",
                           f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"])
    return exe


def test_c_program_compiles_and_links():
    exe = build_program()
    assert os.path.exists(exe)
    # the dynamic symbols the program needs are all exported by the library
    syms = subprocess.run(["nm", "-D", "--undefined-only", exe], capture_output=True, text=True).stdout
    needed = sorted({s.split()[-1] for s in syms.splitlines() if "h3attn_" in s})
    assert needed, syms
    import ctypes
    lib = ctypes.CDLL(h3.LIB_PATH)
    for n in needed:
        assert hasattr(lib, n), n


@pytest.mark.gpu
def test_c_program_matches_the_python_binding(tmp_path):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    exe = build_program()
    w = synth.WORKLOADS["fixed_q128_kv192"]
    x = synth.make_inputs(w)
    inp = tmp_path / "in.bin"
    with open(inp, "wb") as f:
        f.write(struct.pack("<4if", w.B, w.Tq, w.Tkv, w.H, w.scale))
        for n in ("q", "k", "v"):
            f.write(np.ascontiguousarray(x[n]).tobytes())
    outp = tmp_path / "out.bin"
    r = subprocess.run([exe, str(inp), str(outp)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    got = np.fromfile(outp, dtype=np.uint16).reshape(w.B, w.Tq, w.H, w.D)

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)

    out = torch.empty(w.B, w.Tq, w.H, w.D, dtype=torch.bfloat16, device="cuda")
    ws = h3.new_workspace(w.B, w.Tq, w.Tkv, w.H)
    h3.h3attn_forward_ex(dev(x["q"]), dev(x["k"]), dev(x["v"]), w.scale, out, ws)
    assert h3.h3attn_check_status(ws) == h3.OK
    ref = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, ref)


@pytest.mark.gpu
def test_c_program_runs_again_after_a_device_reset(tmp_path):
    """The program runs the forward pass, resets the device (a new context: every
    allocation and every kernel attribute of the old one is gone) and runs it again: the
    library must set its kernels' shared-memory attributes for the new context, and the
    second output must equal the first (the program compares them) and the usual bytes."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    exe = build_program()
    w = synth.WORKLOADS["fixed_q128_kv192"]
    x = synth.make_inputs(w)
    inp = tmp_path / "in.bin"
    with open(inp, "wb") as f:
        f.write(struct.pack("<4if", w.B, w.Tq, w.Tkv, w.H, w.scale))
        for n in ("q", "k", "v"):
            f.write(np.ascontiguousarray(x[n]).tobytes())
    plain, again = tmp_path / "plain.bin", tmp_path / "again.bin"
    r = subprocess.run([exe, str(inp), str(plain)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([exe, str(inp), str(again), "reset"], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "after a device reset" in r.stdout
    assert np.array_equal(np.fromfile(again, dtype=np.uint16), np.fromfile(plain, dtype=np.uint16))

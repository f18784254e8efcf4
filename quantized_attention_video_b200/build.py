"""Build libh3attn.so in-tree with nvcc for sm_100a.

    python -m quantized_attention_video_b200.build [--verbose]

Compiles every .cu under csrc/ into one shared library next to this file.
``-Xptxas -v`` prints registers, spills and shared memory per kernel.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SO = os.path.join(PKG, "libh3attn.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
    "-shared", "-Xptxas", "-v",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))


def needs_build() -> bool:
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    deps = sources() + glob.glob(os.path.join(PKG, "csrc", "*.cuh")) + glob.glob(os.path.join(PKG, "csrc", "*.h")) \
        + [os.path.join(ROOT, "include", "h3attn.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return SO
    tmp = SO + ".tmp"
    cmd = [NVCC] + FLAGS + ["-o", tmp] + sources()
    r = subprocess.run(cmd, capture_output=True, text=True)
    log = r.stdout + r.stderr
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + log)
    if verbose:
        print(log)
    with open(os.path.join(PKG, "ptxas_resources.txt"), "w") as f:
        f.write(log)
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(SO)

"""Build the CUDA library in-tree: w4a4_diffusion_model_b200/libsvdq.so.

    python -m w4a4_diffusion_model_b200.build

Compiles the single translation unit csrc/svdq_api.cu for sm_100a with nvcc
(cross-compiles without a GPU).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "svdq_api.cu")
OUT = os.path.join(HERE, "libsvdq.so")


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def command(out: str = OUT, extra: list[str] | None = None) -> list[str]:
    return [
        nvcc(), "-std=c++17", "-O3", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "--shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
        "-I", os.path.join(ROOT, "include"), "-I", os.path.join(HERE, "csrc"),
        "-o", out, SRC, "-lcudart",
    ] + (extra or [])


def sources() -> list[str]:
    d = os.path.join(HERE, "csrc")
    return [os.path.join(d, f) for f in sorted(os.listdir(d))] + [os.path.join(ROOT, "include", "svdq.h")]


def up_to_date(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    if not force and up_to_date():
        return OUT
    cmd = command(extra=extra)
    if verbose:
        print(" ".join(cmd), flush=True)
    tmp = OUT + ".tmp"
    cmd[cmd.index(OUT)] = tmp
    subprocess.run(cmd, check=True)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)

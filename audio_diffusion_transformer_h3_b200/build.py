"""Builds libh3attn.so in-tree with nvcc for sm_100a.

    python audio_diffusion_transformer_h3_b200/build.py [--verbose]

The library is written next to this file so that it travels with the
source tree; ``audio_diffusion_transformer_h3_b200`` loads it from there.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libh3attn.so")

SOURCES = [os.path.join(CSRC, "h3attn.cu"), os.path.join(CSRC, "h3attn_static.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("sm100.cuh", "rope.cuh", "attn_fwd.cuh", "attn_sage.cuh", "qkv_gemm.cuh")] + [
    os.path.join(INCLUDE, "h3attn.h")]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(verbose: bool = False) -> list[str]:
    cmd = [nvcc(), "-O3", "-std=c++17", "-lineinfo",
           "-gencode", "arch=compute_100a,code=sm_100a",
           "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, "-I", CSRC,
           "-o", LIB] + SOURCES
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS if os.path.exists(d))


def build(force: bool = False, verbose: bool = False) -> str:
    if force or not up_to_date():
        res = subprocess.run(command(verbose), capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
        if verbose:
            sys.stdout.write(res.stdout + res.stderr)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)

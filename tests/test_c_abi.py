"""The header is plain C: a C99 program built with gcc against include/h3attn.h
and linked with libh3attn.so runs the host-only calls and the argument checks
(tests/c/abi_host.c). No GPU is needed."""

import os
import shutil
import subprocess

import pytest

import audio_diffusion_transformer_h3_b200 as h3

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_program_uses_the_abi(tmp_path):
    exe = tmp_path / "abi_host"
    libdir = os.path.dirname(h3.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host.c"),
                    "-L", libdir, "-lh3attn", "-Wl,-rpath," + libdir, "-lm", "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert "c abi ok" in out.stdout

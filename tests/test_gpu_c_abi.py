"""The C ABI used from plain C (tests/c_abi_smoke.c): include/moe.h and
libmoe_b200.so only, device buffers from cudaMalloc, no Python in between."""
import os
import shutil
import subprocess

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
PKG = os.path.join(ROOT, "mixture_experts_ffn_token_b200")


def test_c_program_drives_the_library(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "c_abi_smoke")
    subprocess.run([nvcc, "-Wno-deprecated-gpu-targets", "-o", exe, os.path.join(HERE, "c_abi_smoke.c"),
                    "-I", os.path.join(ROOT, "include"), "-L", PKG, "-lmoe_b200", "-Xlinker", f"-rpath={PKG}",
                    "-lcudart"], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip().endswith("ok"), r.stdout

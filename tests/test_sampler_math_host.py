"""The CUDA sampler's integer arithmetic (mul_le_shift32, pi_free,
quantise_w from csrc/ab_sample.cuh, compiled for the host) against exact
128-bit integer arithmetic on ~10 million random and edge-case inputs,
including operand ranges far beyond what real P rows produce.  Runs on the
CPU: nvcc compiles the header's host-callable functions for the host."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_sampler_integer_math_is_exact(tmp_path):
    nvcc = shutil.which("nvcc") or ("/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else None)
    if nvcc is None:
        pytest.skip("nvcc not available")
    exe = tmp_path / "sampler_math_host"
    subprocess.check_call([nvcc, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-I", os.path.join(ROOT, "block_sparse_attention_queries_b200", "csrc"),
                           "-I", os.path.join(ROOT, "include"), "-o", str(exe),
                           os.path.join(ROOT, "tests", "cuda", "sampler_math_host.cu")])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout[-2000:]
    assert "mismatches 0" in out.stdout

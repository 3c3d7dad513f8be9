"""Host-side checks of pure integer logic of the CUDA path, compiled for the
host by nvcc (the headers' host-callable functions; no GPU needed):

* the sampler's integer arithmetic (mul_le_shift32, pi_free, quantise_w from
  csrc/ab_sample.cuh) against exact 128-bit integer arithmetic on ~11.6
  million random and edge-case inputs, including operand ranges far beyond
  what real P rows produce;
* the attention kernel's merged tile order (Merge in csrc/ab_attention.cuh)
  for every pair of stream lengths up to 96."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_host_check(tmp_path, name):
    nvcc = shutil.which("nvcc") or ("/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else None)
    if nvcc is None:
        pytest.skip("nvcc not available")
    exe = tmp_path / name
    subprocess.check_call([nvcc, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-I", os.path.join(ROOT, "block_sparse_attention_queries_b200", "csrc"),
                           "-I", os.path.join(ROOT, "include"), "-o", str(exe),
                           os.path.join(ROOT, "tests", "cuda", name + ".cu")])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout[-2000:]
    return out.stdout


def test_sampler_integer_math_is_exact(tmp_path):
    assert "mismatches 0" in _run_host_check(tmp_path, "sampler_math_host")


def test_attention_merged_tile_order(tmp_path):
    assert "violations 0" in _run_host_check(tmp_path, "merge_host")

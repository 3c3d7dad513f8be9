"""The attention kernel's FMA-pipe exp2 (a Cody-Waite split with a fitted
cubic, `exp2_poly2` in ab_ptx.cuh) against CUDA's exp2f on the same device:
relative error below 1e-4 over the kernel's input range [-125, 8]."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_exp2_poly_matches_exp2f():
    so = os.path.join(HERE, "cuda", "exp2_poly.so")
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared", "-Xcompiler",
                           "-fPIC", "-I", os.path.join(ROOT, "include"), "-I",
                           os.path.join(ROOT, "block_sparse_attention_queries_b200", "csrc"), "-o", so,
                           os.path.join(HERE, "cuda", "exp2_poly.cu")])
    lib = ctypes.CDLL(so)
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-125, 8, 1 << 20), np.arange(-125, 9, 0.25),
                        np.array([0.0, -0.5, 0.5, -0.49999997, 7.9999995])]).astype(np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(1.0))
    poly = np.zeros_like(x)
    ref = np.zeros_like(x)
    assert lib.exp2_poly_eval(x.ctypes.data_as(ctypes.c_void_p), poly.ctypes.data_as(ctypes.c_void_p),
                              ref.ctypes.data_as(ctypes.c_void_p), x.size) == 0
    rel = np.abs(poly.astype(np.float64) / ref.astype(np.float64) - 1)
    assert rel.max() < 1e-4, (rel.max(), x[rel.argmax()])
    # below the clamp the result stays a tiny normal number
    y = np.array([-126.0, -200.0, -1e30, -130.5], np.float32)
    p2 = np.zeros_like(y)
    r2 = np.zeros_like(y)
    lib.exp2_poly_eval(y.ctypes.data_as(ctypes.c_void_p), p2.ctypes.data_as(ctypes.c_void_p),
                       r2.ctypes.data_as(ctypes.c_void_p), y.size)
    assert (p2 > 0).all() and (p2 <= 2.0 ** -124).all()

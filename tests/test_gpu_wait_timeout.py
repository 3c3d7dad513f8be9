"""Failure detection without a fault: the library's bounded mbarrier waits
(the ones every kernel role uses) on a barrier that nothing completes.  The
first wait gives up after its 2 s limit, writes AB_ERR_TIMEOUT (5) into the
device error word and raises the CTA's abort flag; a second role waiting on
the same barrier returns at once through the flag; the drain form gives up
after the limit too.  The kernel then ends normally and the context stays
usable."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
AB_ERR_TIMEOUT = 5


def test_bounded_waits_time_out_and_report():
    so = os.path.join(HERE, "cuda", "wait_timeout.so")
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared", "-Xcompiler",
                           "-fPIC", "-I", os.path.join(ROOT, "include"), "-I",
                           os.path.join(ROOT, "block_sparse_attention_queries_b200", "csrc"), "-o", so,
                           os.path.join(HERE, "cuda", "wait_timeout.cu")])
    lib = ctypes.CDLL(so)
    out = np.zeros(8, np.int32)
    assert lib.wait_timeout_probe(out.ctypes.data_as(ctypes.c_void_p)) == 0
    ok0, ms0, abort_flag, ms1, ok1, drain_ok, err = (int(v) for v in out[:7])
    assert ok0 == 0 and abort_flag == 1 and err == AB_ERR_TIMEOUT
    assert 1900 <= ms0 <= 4000, ms0        # gave up at the 2 s limit
    assert ok1 == 0 and ms1 < 100, ms1      # the other role left through the abort flag
    assert drain_ok == 0                    # the drain wait is bounded as well
    # the context is still usable
    import torch
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum().item()) == 8.0

"""ab_select_static: the selector variant whose scratch is the library's own
fixed device array, for callers that cannot allocate device memory (plugins
under a host framework's memory planner, code that must not block on
cudaMalloc).  Checked through the C ABI against ab_select with a
caller-supplied workspace, on two calls in a row (the array keeps the first
call's contents, which the second must not depend on).  This file is
collected last on purpose."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_sparse_attention_queries_b200 as ab  # noqa: E402
from block_sparse_attention_queries_b200.synthetic import WORKLOADS, make_workload_qkv  # noqa: E402

AB_ERR_WORKSPACE = 6


def _select_static(lib, p, Q, K, dev):
    P = torch.full((p.B, p.H, p.Nq, p.Nkv), float("nan"), dtype=torch.float32, device=dev)
    cent = torch.full((p.B, p.H, p.Nq, p.C, p.d), float("nan"), dtype=torch.float32, device=dev)
    cnt = torch.full((p.B, p.H, p.Nq, p.C), -1, dtype=torch.int32, device=dev)
    st = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    s = lib.ab_select_static(ctypes.byref(p.c()), ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()),
                             ctypes.c_void_p(P.data_ptr()), ctypes.c_void_p(cent.data_ptr()),
                             ctypes.c_void_p(cnt.data_ptr()), st)
    assert s == 0, ab.status_string(s)
    return P, cent, cnt


@pytest.mark.parametrize("wname", ["small", "tiny"])
def test_select_static_matches_workspace_select(wname):
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    dev = torch.device("cuda:0")
    lib = ab.lib()
    w = WORKLOADS[wname]
    p = ab.Params.of(w)
    Qc, Kc, _ = make_workload_qkv(w)
    Q, K = Qc.to(dev), Kc.to(dev)
    P_ref, c_ref, n_ref = ab.ab_select(p, Q, K, want_centroids=True)
    for _ in range(2):
        P, cent, cnt = _select_static(lib, p, Q, K, dev)
        torch.cuda.synchronize()
        assert ab.device_error(dev) == 0
        # same kernels on the same inputs: identical results
        np.testing.assert_array_equal(P.cpu().numpy(), P_ref.cpu().numpy())
        np.testing.assert_array_equal(cent.cpu().numpy(), c_ref.cpu().numpy())
        np.testing.assert_array_equal(cnt.cpu().numpy(), n_ref.cpu().numpy())


def test_select_static_rejects_problems_beyond_the_limit():
    lib = ab.lib()
    # HunyuanVideo-720p layer: 91 MB of scratch > 48 MiB; rejected before any launch
    w = WORKLOADS["hunyuan720"]
    p = ab.Params.of(w)
    assert ab.workspace_size(p) > 48 * 1024 * 1024
    fake = ctypes.c_void_p(0x10000)
    s = lib.ab_select_static(ctypes.byref(p.c()), fake, fake, fake, None, None, None)
    assert s == AB_ERR_WORKSPACE

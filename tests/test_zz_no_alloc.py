"""ab_select_static: the selector variant whose scratch is the library's own
fixed device array, for callers that cannot allocate device memory (plugins
under a host framework's memory planner, code that must not block on
cudaMalloc).  Checked through the C ABI against ab_select with a
caller-supplied workspace, on two calls in a row that follow a call on a
different problem (the array keeps each call's contents, which the next call
must not depend on).  This file is collected last on purpose."""
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


def _dev():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    return torch.device("cuda:0")


def _case(wname, seed, dev):
    w = WORKLOADS[wname]
    p = ab.Params.of(w)
    Qc, Kc, _ = make_workload_qkv(w, seed=seed)
    return p, Qc.to(dev), Kc.to(dev)


@pytest.mark.parametrize("wname,other", [("small", "tiny"), ("tiny", "small")])
def test_select_static_matches_workspace_select(wname, other):
    # Each checked call follows a call on a different problem (other shape,
    # other inputs), so what that call left in the shared array differs from
    # what this one needs; then the check is repeated on a second call in a row.
    dev = _dev()
    lib = ab.lib()
    p, Q, K = _case(wname, 1234, dev)
    P_ref, c_ref, n_ref = ab.ab_select(p, Q, K, want_centroids=True)
    po, Qo, Ko = _case(other, 777, dev)
    _select_static(lib, po, Qo, Ko, dev)
    for _ in range(2):
        P, cent, cnt = _select_static(lib, p, Q, K, dev)
        torch.cuda.synchronize()
        assert ab.device_error(dev) == 0
        # same kernels on the same inputs: identical results
        np.testing.assert_array_equal(P.cpu().numpy(), P_ref.cpu().numpy())
        np.testing.assert_array_equal(cent.cpu().numpy(), c_ref.cpu().numpy())
        np.testing.assert_array_equal(cnt.cpu().numpy(), n_ref.cpu().numpy())


def test_select_static_rejects_problems_beyond_the_limit():
    dev = _dev()
    lib = ab.lib()
    # HunyuanVideo-720p layer: 91 MB of scratch > 48 MiB; rejected before any
    # launch (the buffers are real, small device tensors: nothing reads them)
    w = WORKLOADS["hunyuan720"]
    p = ab.Params.of(w)
    assert ab.workspace_size(p) > 48 * 1024 * 1024
    buf = torch.zeros(1024, dtype=torch.float32, device=dev)
    ptr = ctypes.c_void_p(buf.data_ptr())
    st = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    s = lib.ab_select_static(ctypes.byref(p.c()), ptr, ptr, ptr, None, None, st)
    assert s == AB_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.equal(buf, torch.zeros_like(buf))

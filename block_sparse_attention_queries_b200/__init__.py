"""AB-Attention (Accurate Block Attention) hot path on NVIDIA B200.

Python binding of the C ABI in ``include/ab.h`` (library ``libab.so`` in this
package).  This module only marshals arguments: it checks tensor shapes and
dtypes, allocates outputs with torch on the caller's device and passes raw
pointers and the current CUDA stream to the library.  Every step of the path
runs in the library's CUDA kernels; there is no CPU fallback, and calling any
op without the built library raises ``RuntimeError``.

Names follow the C ABI: ``ab_select`` (IBCS), ``ab_sample`` (SIP),
``ab_attention`` (the packed 1/pi-weighted sparse attention),
``ab_attention_dense``, ``ab_forward`` and ``ab_forward_host``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libab.so")

AB_OK = 0
STATUS_NAMES = {0: "AB_OK", 1: "AB_ERR_INVALID_ARG", 2: "AB_ERR_UNSUPPORTED", 3: "AB_ERR_CUDA",
                4: "AB_ERR_CAPACITY", 5: "AB_ERR_TIMEOUT", 6: "AB_ERR_WORKSPACE"}

# every symbol include/ab.h declares
EXPORTS = ("ab_budget", "ab_workspace_size", "ab_select", "ab_sample", "ab_sample_systematic", "ab_sample_topk", "ab_attention",
           "ab_attention_dense", "ab_forward", "ab_forward_host", "ab_get_device_error",
           "ab_status_string", "ab_select_static", "ab_forward_slice", "ab_select_sample")


class AbError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class ab_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("L", ctypes.c_int32),
                ("d", ctypes.c_int32), ("q_block", ctypes.c_int32), ("kv_block", ctypes.c_int32),
                ("C", ctypes.c_int32), ("kmeans_iters", ctypes.c_int32),
                ("keep_ratio", ctypes.c_float), ("L_kv", ctypes.c_int32), ("seed", ctypes.c_uint64)]


@dataclass(frozen=True)
class Params:
    """Problem description (mirrors ``ab_params``).  ``L`` is the number of
    queries per (b, h); ``L_kv`` the number of keys and values (0: the same as
    ``L``, i.e. self-attention)."""

    B: int
    H: int
    L: int
    d: int
    q_block: int = 128
    kv_block: int = 16
    C: int = 8
    kmeans_iters: int = 3
    keep_ratio: float = 0.1
    seed: int = 42
    L_kv: int = 0

    @property
    def Lk(self) -> int:
        return self.L_kv if self.L_kv > 0 else self.L

    @property
    def Nq(self) -> int:
        return -(-self.L // self.q_block)

    @property
    def Nkv(self) -> int:
        return -(-self.Lk // self.kv_block)

    def c(self) -> ab_params:
        return ab_params(self.B, self.H, self.L, self.d, self.q_block, self.kv_block, self.C,
                         self.kmeans_iters, float(self.keep_ratio), int(self.L_kv),
                         int(self.seed) & (2**64 - 1))

    @staticmethod
    def of(w, seed: int = 42, **kw) -> "Params":
        """From a ``synthetic.Workload``."""
        args = dict(B=w.B, H=w.H, L=w.L, d=w.d, q_block=w.q_block, kv_block=w.kv_block, C=w.C,
                    kmeans_iters=w.kmeans_iters, keep_ratio=w.keep_ratio, seed=seed,
                    L_kv=w.Lk if w.Lk != w.L else 0)
        args.update(kw)
        return Params(**args)


_lib = None


def lib(path: str = LIB_PATH):
    """The loaded ``libab.so``; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"libab.so not built ({path}); run block_sparse_attention_queries_b200/build.py")
        L = ctypes.CDLL(path)
        P = ctypes.POINTER(ab_params)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        L.ab_budget.argtypes = [P]
        L.ab_budget.restype = ctypes.c_int32
        L.ab_workspace_size.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
        L.ab_select.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
        L.ab_sample.argtypes = [P, vp, vp, vp, vp, vp]
        L.ab_sample_topk.argtypes = [P, vp, vp, vp, vp, vp]
        L.ab_sample_systematic.argtypes = [P, vp, vp, vp, vp, vp]
        L.ab_attention.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp]
        L.ab_attention_dense.argtypes = [P, vp, vp, vp, vp, vp]
        L.ab_forward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.ab_forward_host.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.ab_select_sample.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.ab_forward_slice.argtypes = [P, ctypes.c_int32, ctypes.c_int32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                       vp]
        L.ab_select_static.argtypes = [P, vp, vp, vp, vp, vp, vp]
        L.ab_get_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
        L.ab_status_string.argtypes = [ctypes.c_int]
        L.ab_status_string.restype = ctypes.c_char_p
        for name in ("ab_workspace_size", "ab_select", "ab_sample", "ab_sample_systematic", "ab_sample_topk", "ab_attention",
                     "ab_attention_dense",
                     "ab_forward", "ab_forward_host", "ab_get_device_error", "ab_select_static",
                     "ab_forward_slice", "ab_select_sample"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != AB_OK:
        raise AbError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check_bf16(t, shape):
    import torch
    if t.dtype != torch.bfloat16 or tuple(t.shape) != shape or not t.is_contiguous():
        raise ValueError(f"expected contiguous bf16 {list(shape)}, got {t.dtype} {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")


def _check_qkv(p: Params, Q, *kv):
    """Q (and O) are [B, H, L, d]; K and V are [B, H, Lk, d]."""
    _check_bf16(Q, (p.B, p.H, p.L, p.d))
    for t in kv:
        _check_bf16(t, (p.B, p.H, p.Lk, p.d))


def budget(p: Params) -> int:
    return int(lib().ab_budget(ctypes.byref(p.c())))


def workspace_size(p: Params) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().ab_workspace_size(ctypes.byref(p.c()), ctypes.byref(n)), "ab_workspace_size")
    return int(n.value)


def alloc_workspace(p: Params, device):
    import torch
    return torch.empty(workspace_size(p), dtype=torch.uint8, device=device)


def ab_select(p: Params, Q, K, workspace=None, want_centroids=False):
    """IBCS: returns P [B,H,Nq,Nkv] fp32 (and centroids [B,H,Nq,C,d] fp32, counts [B,H,Nq,C] int32)."""
    import torch
    _check_qkv(p, Q, K)
    dev = Q.device
    P = torch.empty(p.B, p.H, p.Nq, p.Nkv, dtype=torch.float32, device=dev)
    cent = torch.empty(p.B, p.H, p.Nq, p.C, p.d, dtype=torch.float32, device=dev) if want_centroids else None
    cnt = torch.empty(p.B, p.H, p.Nq, p.C, dtype=torch.int32, device=dev) if want_centroids else None
    ws = alloc_workspace(p, dev) if workspace is None else workspace
    _check(lib().ab_select(ctypes.byref(p.c()), _ptr(Q), _ptr(K), _ptr(P), _ptr(cent), _ptr(cnt), _ptr(ws),
                           ws.numel(), _stream(dev)), "ab_select")
    return (P, cent, cnt) if want_centroids else P


def ab_select_static(p: Params, Q, K, want_centroids=False):
    """ab_select with the library's own fixed device scratch: no workspace is
    allocated (the outputs still are, here, by torch).  For callers that
    cannot allocate device memory; see include/ab.h for the size limit and the
    rule that overlapping calls race."""
    import torch
    _check_qkv(p, Q, K)
    dev = Q.device
    P = torch.empty(p.B, p.H, p.Nq, p.Nkv, dtype=torch.float32, device=dev)
    cent = torch.empty(p.B, p.H, p.Nq, p.C, p.d, dtype=torch.float32, device=dev) if want_centroids else None
    cnt = torch.empty(p.B, p.H, p.Nq, p.C, dtype=torch.int32, device=dev) if want_centroids else None
    _check(lib().ab_select_static(ctypes.byref(p.c()), _ptr(Q), _ptr(K), _ptr(P), _ptr(cent), _ptr(cnt),
                                  _stream(dev)), "ab_select_static")
    return (P, cent, cnt) if want_centroids else P


def _list_outputs(p: Params, P, out):
    """Checks P and returns (idx, pi_q32, count): `out` if given (checked), else new zeroed tensors."""
    import torch
    if P.dtype != torch.float32 or tuple(P.shape) != (p.B, p.H, p.Nq, p.Nkv) or not P.is_contiguous():
        raise ValueError("P must be contiguous fp32 [B,H,Nq,Nkv]")
    dev = P.device
    if out is None:
        return (torch.zeros(p.B, p.H, p.Nq, p.Nkv, dtype=torch.int32, device=dev),
                torch.zeros(p.B, p.H, p.Nq, p.Nkv, dtype=torch.int32, device=dev),
                torch.zeros(p.B, p.H, p.Nq, dtype=torch.int32, device=dev))
    for t, shape in zip(out, ((p.B, p.H, p.Nq, p.Nkv), (p.B, p.H, p.Nq, p.Nkv), (p.B, p.H, p.Nq))):
        if t.dtype not in (torch.int32, torch.uint32) or tuple(t.shape) != shape or not t.is_contiguous() \
                or t.device != dev:
            raise ValueError(f"list output must be contiguous int32 {shape} on {dev}")
    return tuple(out)


def _lists_call(fn_name, p: Params, P, out=None):
    idx, piq, cnt = _list_outputs(p, P, out)
    _check(getattr(lib(), fn_name)(ctypes.byref(p.c()), _ptr(P), _ptr(idx), _ptr(piq), _ptr(cnt),
                                   _stream(P.device)), fn_name)
    return idx, piq, cnt


def ab_select_sample(p: Params, Q, K, workspace=None, out=None):
    """ab_select then ab_sample in one call (the scoring kernel samples the
    rows it scores when rows have at most 2048 KV blocks); returns
    (P, idx, pi_q32, count), bit-identical to the two calls in a row.
    `out` = (P, idx, pi_q32, count) writes into caller-owned tensors."""
    import torch
    _check_qkv(p, Q, K)
    if out is None:
        P = torch.empty(p.B, p.H, p.Nq, p.Nkv, dtype=torch.float32, device=Q.device)
        idx, piq, cnt = _list_outputs(p, P, None)
    else:
        P, idx, piq, cnt = out
        if P.dtype != torch.float32 or tuple(P.shape) != (p.B, p.H, p.Nq, p.Nkv) or not P.is_contiguous():
            raise ValueError("P must be contiguous float32 [B, H, Nq, Nkv]")
        idx, piq, cnt = _list_outputs(p, P, (idx, piq, cnt))
    ws = alloc_workspace(p, Q.device) if workspace is None else workspace
    _check(lib().ab_select_sample(ctypes.byref(p.c()), _ptr(Q), _ptr(K), _ptr(P), _ptr(idx), _ptr(piq), _ptr(cnt),
                                  _ptr(ws), ws.numel(), _stream(Q.device)), "ab_select_sample")
    return P, idx, piq, cnt


def ab_sample(p: Params, P, out=None):
    """SIP: returns idx [B,H,Nq,Nkv] int32, pi_q32 [B,H,Nq,Nkv] uint32 (as int32 storage), count [B,H,Nq].
    `out` = (idx, pi_q32, count) writes into caller-owned tensors instead."""
    return _lists_call("ab_sample", p, P, out)


def ab_sample_systematic(p: Params, P, out=None):
    """Systematic sampling with SIP's inclusion probabilities: same outputs as ab_sample."""
    return _lists_call("ab_sample_systematic", p, P, out)


def ab_sample_topk(p: Params, P, out=None):
    """Truncation (top-Kb by P, ties to the lower block, pi = 1): same outputs as ab_sample."""
    return _lists_call("ab_sample_topk", p, P, out)


def ab_attention(p: Params, Q, K, V, idx, pi_q32, count, out=None):
    """Packed 1/pi-weighted block-sparse attention; Q [B,H,L,d], K and V
    [B,H,Lk,d]; returns O [B,H,L,d] bf16."""
    import torch
    _check_qkv(p, Q, K, V)
    for t, shape in ((idx, (p.B, p.H, p.Nq, p.Nkv)), (pi_q32, (p.B, p.H, p.Nq, p.Nkv)), (count, (p.B, p.H, p.Nq))):
        if t.dtype not in (torch.int32, torch.uint32) or tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"list tensor must be contiguous int32 {shape}")
    O = torch.empty_like(Q) if out is None else out
    _check_bf16(O, (p.B, p.H, p.L, p.d))
    _check(lib().ab_attention(ctypes.byref(p.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(pi_q32),
                              _ptr(count), _ptr(O), _stream(Q.device)), "ab_attention")
    return O


def ab_attention_dense(p: Params, Q, K, V, out=None):
    """Dense softmax(QK^T/sqrt(d))V with the same kernel family; returns O."""
    import torch
    _check_qkv(p, Q, K, V)
    O = torch.empty_like(Q) if out is None else out
    _check_bf16(O, (p.B, p.H, p.L, p.d))
    _check(lib().ab_attention_dense(ctypes.byref(p.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                    _stream(Q.device)), "ab_attention_dense")
    return O


class Buffers:
    """Device buffers of one layer (P, lists, output, workspace)."""

    def __init__(self, p: Params, device):
        import torch
        self.P = torch.empty(p.B, p.H, p.Nq, p.Nkv, dtype=torch.float32, device=device)
        self.idx = torch.zeros(p.B, p.H, p.Nq, p.Nkv, dtype=torch.int32, device=device)
        self.pi_q32 = torch.zeros(p.B, p.H, p.Nq, p.Nkv, dtype=torch.int32, device=device)
        self.count = torch.zeros(p.B, p.H, p.Nq, dtype=torch.int32, device=device)
        self.O = torch.empty(p.B, p.H, p.L, p.d, dtype=torch.bfloat16, device=device)
        self.ws = alloc_workspace(p, device)


def ab_forward(p: Params, Q, K, V, bufs: Buffers | None = None) -> Buffers:
    """ab_select -> ab_sample -> ab_attention on device buffers."""
    _check_qkv(p, Q, K, V)
    b = Buffers(p, Q.device) if bufs is None else bufs
    _check(lib().ab_forward(ctypes.byref(p.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(b.P), _ptr(b.idx),
                            _ptr(b.pi_q32), _ptr(b.count), _ptr(b.O), _ptr(b.ws), b.ws.numel(),
                            _stream(Q.device)), "ab_forward")
    return b


def head_slices(B: int, H: int, world: int):
    """Contiguous near-equal partition of a layer's B * H heads among `world`
    ranks: [(bh0, nbh), ...], rank r taking flattened heads [bh0, bh0 + nbh)
    (the first B*H % world ranks take one head more).  Every rank gets at
    least one head, so world must not exceed B * H."""
    n = B * H
    if not 1 <= world <= n:
        raise ValueError(f"cannot split {n} heads among {world} ranks")
    base, extra = divmod(n, world)
    out, bh0 = [], 0
    for r in range(world):
        nbh = base + (1 if r < extra else 0)
        out.append((bh0, nbh))
        bh0 += nbh
    return out


def slice_rows(p: Params, bh0: int, nbh: int):
    """(b, h, i) in the whole problem of every row of a slice's per-row
    buffers (P, idx, pi_q32: [nbh, Nq, ...]; count: [nbh, Nq]), in their
    order: local row r is row bh0 * Nq + r of the whole [B, H, Nq] layout.
    These are the counters SIP draws a slice's rows with (the library derives
    the same from the slice's first row and the whole problem's H)."""
    out = []
    for lb in range(nbh):
        b, h = divmod(bh0 + lb, p.H)
        out.extend((b, h, i) for i in range(p.Nq))
    return out


def slice_params(p: Params, nbh: int) -> Params:
    """The problem of one slice of nbh heads (B = 1, H = nbh): its buffer
    shapes and workspace size.  The whole problem's Params stay the ones
    passed to ab_forward_slice."""
    from dataclasses import replace
    return replace(p, B=1, H=nbh)


def ab_forward_slice(p: Params, bh0: int, nbh: int, Q, K, V, bufs: Buffers | None = None) -> Buffers:
    """ab_forward on heads [bh0, bh0 + nbh) of the problem `p` (flattened b * H
    + h): Q [1, nbh, L, d], K and V [1, nbh, Lk, d]; the buffers are the
    slice's (Buffers(slice_params(p, nbh))).  The draws use the whole
    problem's counters, so the result equals those heads of ab_forward(p)."""
    ps = slice_params(p, nbh)
    _check_qkv(ps, Q, K, V)
    b = Buffers(ps, Q.device) if bufs is None else bufs
    _check(lib().ab_forward_slice(ctypes.byref(p.c()), int(bh0), int(nbh), _ptr(Q), _ptr(K), _ptr(V), _ptr(b.P),
                                  _ptr(b.idx), _ptr(b.pi_q32), _ptr(b.count), _ptr(b.O), _ptr(b.ws), b.ws.numel(),
                                  _stream(Q.device)), "ab_forward_slice")
    return b


def ab_forward_host(p: Params, Qh, Kh, Vh, Oh, Qd, Kd, Vd, bufs: Buffers, device):
    """Host bf16 Qh [B,H,L,d], Kh and Vh [B,H,Lk,d] -> host out Oh [B,H,L,d];
    Qd/Kd/Vd are device staging buffers of the same shapes."""
    for t, n in ((Qh, p.L), (Kh, p.Lk), (Vh, p.Lk), (Oh, p.L), (Qd, p.L), (Kd, p.Lk), (Vd, p.Lk)):
        if tuple(t.shape) != (p.B, p.H, n, p.d) or not t.is_contiguous():
            raise ValueError(f"expected contiguous [{p.B},{p.H},{n},{p.d}], got {tuple(t.shape)}")
    _check(lib().ab_forward_host(ctypes.byref(p.c()), _ptr(Qh), _ptr(Kh), _ptr(Vh), _ptr(Oh), _ptr(Qd),
                                 _ptr(Kd), _ptr(Vd), _ptr(bufs.P), _ptr(bufs.idx), _ptr(bufs.pi_q32),
                                 _ptr(bufs.count), _ptr(bufs.O), _ptr(bufs.ws), bufs.ws.numel(),
                                 _stream(device)), "ab_forward_host")


def device_error(device=None) -> int:
    """Reads and clears the library's device error word (0 = none)."""
    code = ctypes.c_int32(0)
    _check(lib().ab_get_device_error(_stream(device), ctypes.byref(code)), "ab_get_device_error")
    return int(code.value)


def status_string(code: int) -> str:
    return lib().ab_status_string(int(code)).decode()

"""CPU oracle for the AB-Attention hot path (ctypes binding of ab_oracle.cpp).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The CUDA library never
imports, links or runs anything here, and this module never touches the CUDA
library.

Every array crossing into C is a contiguous numpy array; floating inputs are
the fp32 values of the bfloat16 tensors (exact), outputs are fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ab_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u32p = np.ctypeslib.ndpointer(dtype=np.uint32, flags="C_CONTIGUOUS")
_u64p = np.ctypeslib.ndpointer(dtype=np.uint64, flags="C_CONTIGUOUS")
_ci, _cd, _cu64, _vp = ctypes.c_int, ctypes.c_double, ctypes.c_uint64, ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile liboracle.so with plain g++ (IEEE arithmetic, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-fno-fast-math",
               "-o", _LIB + ".tmp", _SRC]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.orc_philox4x32_10.argtypes = [_u32p, _u32p, _u32p]
        L.orc_dense_rows.argtypes = [_f32p, _f32p, _f32p, _ci, _ci, _ci, _ci, _f64p]
        L.orc_ksum.argtypes = [_f32p, _ci, _ci, _ci, _f64p]
        L.orc_kmeans.argtypes = [_f32p, _ci, _ci, _ci, _ci, _f64p, _i32p, _vp]
        L.orc_kmeans.restype = _ci
        L.orc_block_mass.argtypes = [_f64p, _i32p, _ci, _ci, _f64p, _ci, _ci, _ci, _ci, _f64p]
        L.orc_select_head.argtypes = [_f32p, _f32p, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _vp, _ci,
                                      _f64p, _vp, _vp]
        L.orc_budget.argtypes = [_ci, _cd]
        L.orc_budget.restype = _ci
        L.orc_sip_row.argtypes = [_f32p, _ci, _ci, _cu64, _ci, _ci, _ci, _i32p, _u32p, _i32p, _vp]
        L.orc_sip_row.restype = _ci
        L.orc_topk_row.argtypes = [_f32p, _ci, _ci, _i32p, _u32p, _i32p]
        L.orc_systematic_row.argtypes = [_f32p, _ci, _ci, _cu64, _ci, _ci, _ci, _i32p, _u32p, _i32p]
        L.orc_systematic_row.restype = _ci
        L.orc_systematic_row_u.argtypes = [_f32p, _ci, _ci, _cu64, _i32p, _u32p, _i32p]
        L.orc_systematic_row_u.restype = _ci
        L.orc_topk_row.restype = _ci
        L.orc_ht_sums.argtypes = [_f32p, _f32p, _f32p, _ci, _ci, _ci, _i32p, _u32p, _ci, _cd,
                                  _f64p, _f64p]
        L.orc_ht_attention_block.argtypes = [_f32p, _f32p, _f32p, _ci, _ci, _ci, _ci, _ci, _ci,
                                             _i32p, _u32p, _ci, _f64p]
        _lib = L
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- primitives

def philox4x32_10(ctr, key):
    out = np.zeros(4, np.uint32)
    lib().orc_philox4x32_10(np.asarray(ctr, np.uint32), np.asarray(key, np.uint32), out)
    return out


def budget(Nkv: int, keep_ratio: float) -> int:
    return int(lib().orc_budget(int(Nkv), float(keep_ratio)))


def dense_rows(Q, K, V, row0=0, nrows=None):
    """Dense softmax(QK^T/sqrt(d))V for rows [row0, row0+nrows) of one head.

    Q is [L, d]; K and V are [Lk, d] (Lk = L for self-attention)."""
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    L, d = Q.shape
    Lk = K.shape[0]
    assert V.shape == K.shape and K.shape[1] == d
    nrows = L - row0 if nrows is None else nrows
    assert 0 <= row0 and row0 + nrows <= L
    O = np.zeros((nrows, d), np.float64)
    lib().orc_dense_rows(Q, K, V, Lk, d, row0, nrows, O)
    return O


def ksum(K, kv_block):
    K = _f32(K)
    L, d = K.shape
    out = np.zeros((-(-L // kv_block), d), np.float64)
    lib().orc_ksum(K, L, d, kv_block, out)
    return out


def kmeans(Qb, C, iters, return_assign=False):
    Qb = _f32(Qb)
    n, d = Qb.shape
    mu = np.zeros((C, d), np.float64)
    counts = np.zeros(C, np.int32)
    assign = np.zeros(n, np.int32)
    lib().orc_kmeans(Qb, n, d, C, iters, mu, counts, _ptr(assign))
    return (mu, counts, assign) if return_assign else (mu, counts)


def block_mass(mu, counts, n_i, Ksum, L, kv_block):
    mu = np.ascontiguousarray(mu, np.float64)
    counts = np.ascontiguousarray(counts, np.int32)
    Ksum = np.ascontiguousarray(Ksum, np.float64)
    C, d = mu.shape
    Nkv = Ksum.shape[0]
    P = np.zeros(Nkv, np.float64)
    lib().orc_block_mass(mu, counts, C, n_i, Ksum, Nkv, L, kv_block, d, P)
    return P


def select_head(Q, K, q_block, kv_block, C, iters, rows=None, want_centroids=False):
    """IBCS for one (b, h): returns P [nrows, Nkv] (and mu, counts).

    Q is [L, d] (query blocks), K is [Lk, d] (KV blocks; Lk = L for
    self-attention)."""
    Q, K = _f32(Q), _f32(K)
    L, d = Q.shape
    Lk = K.shape[0]
    assert K.shape[1] == d
    Nq, Nkv = -(-L // q_block), -(-Lk // kv_block)
    rows_a = None if rows is None else np.ascontiguousarray(rows, np.int32)
    nrows = Nq if rows is None else len(rows_a)
    P = np.zeros((nrows, Nkv), np.float64)
    mu = np.zeros((nrows, C, d), np.float64) if want_centroids else None
    cnt = np.zeros((nrows, C), np.int32) if want_centroids else None
    lib().orc_select_head(Q, K, L, Lk, d, q_block, kv_block, C, iters, _ptr(rows_a), nrows, P,
                          _ptr(mu), _ptr(cnt))
    return (P, mu, cnt) if want_centroids else P


def sip_row(P_row, Kb, seed, b, h, i, want_pi=False):
    """SIP on one fp32 row: returns idx, pi_q32, count (and the 64-bit Pi)."""
    P_row = _f32(P_row)
    Nkv = P_row.shape[0]
    idx = np.zeros(Nkv, np.int32)
    pq = np.zeros(Nkv, np.uint32)
    cnt = np.zeros(1, np.int32)
    Pi = np.zeros(Nkv, np.uint64) if want_pi else None
    lib().orc_sip_row(P_row, Nkv, int(Kb), ctypes.c_uint64(int(seed)), b, h, i, idx, pq, cnt,
                      _ptr(Pi))
    n = int(cnt[0])
    out = (idx[:n].copy(), pq[:n].copy(), n)
    return out + (Pi,) if want_pi else out


def systematic_row(P_row, Kb, seed, b, h, i):
    """Systematic sampling with SIP's inclusion probabilities on one fp32 row: idx, pi_q32, count."""
    P_row = _f32(P_row)
    Nkv = P_row.shape[0]
    idx = np.zeros(Nkv, np.int32)
    pq = np.zeros(Nkv, np.uint32)
    cnt = np.zeros(1, np.int32)
    lib().orc_systematic_row(P_row, Nkv, int(Kb), ctypes.c_uint64(int(seed)), b, h, i, idx, pq, cnt)
    n = int(cnt[0])
    return idx[:n].copy(), pq[:n].copy(), n


def systematic_row_u(P_row, Kb, U):
    """The systematic selection for an explicit offset U in [0, 2^32)."""
    P_row = _f32(P_row)
    Nkv = P_row.shape[0]
    idx = np.zeros(Nkv, np.int32)
    pq = np.zeros(Nkv, np.uint32)
    cnt = np.zeros(1, np.int32)
    lib().orc_systematic_row_u(P_row, Nkv, int(Kb), ctypes.c_uint64(int(U)), idx, pq, cnt)
    n = int(cnt[0])
    return idx[:n].copy(), pq[:n].copy(), n


def topk_row(P_row, Kb):
    """Truncation on one fp32 row: the Kb largest P (ties to the lower j), ascending, pi = 1."""
    P_row = _f32(P_row)
    Nkv = P_row.shape[0]
    idx = np.zeros(Nkv, np.int32)
    pq = np.zeros(Nkv, np.uint32)
    cnt = np.zeros(1, np.int32)
    lib().orc_topk_row(P_row, Nkv, int(Kb), idx, pq, cnt)
    n = int(cnt[0])
    return idx[:n].copy(), pq[:n].copy(), n


def sip(P, Kb, seed, b_index=None):
    """SIP over P [B, H, Nq, Nkv] fp32: full-capacity idx/pi arrays and counts."""
    P = _f32(P)
    B, H, Nq, Nkv = P.shape
    idx = np.zeros((B, H, Nq, Nkv), np.int32)
    pq = np.zeros((B, H, Nq, Nkv), np.uint32)
    count = np.zeros((B, H, Nq), np.int32)
    L = lib()
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                c = np.zeros(1, np.int32)
                ii = np.zeros(Nkv, np.int32)
                pp = np.zeros(Nkv, np.uint32)
                L.orc_sip_row(np.ascontiguousarray(P[b, h, i]), Nkv, int(Kb),
                              ctypes.c_uint64(int(seed)), b, h, i, ii, pp, c, None)
                n = int(c[0])
                idx[b, h, i, :n] = ii[:n]
                pq[b, h, i, :n] = pp[:n]
                count[b, h, i] = n
    return idx, pq, count


def ht_sums(q, K, V, kv_block, idx, pi_q32, shift):
    q, K, V = _f32(q), _f32(K), _f32(V)
    L, d = K.shape
    idx = np.ascontiguousarray(idx, np.int32)
    pq = np.ascontiguousarray(pi_q32, np.uint32)
    num = np.zeros(d, np.float64)
    den = np.zeros(1, np.float64)
    lib().orc_ht_sums(q, K, V, L, d, kv_block, idx, pq, len(idx), float(shift), num, den)
    return num, float(den[0])


def ht_attention_block(Q, K, V, q_block, kv_block, i, idx, pi_q32, count):
    """Reweighted attention of query block i: Q [L, d], K and V [Lk, d]."""
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    L, d = Q.shape
    Lk = K.shape[0]
    assert V.shape == K.shape and K.shape[1] == d
    n_i = min(q_block, L - i * q_block)
    idx = np.ascontiguousarray(idx[:count], np.int32)
    pq = np.ascontiguousarray(pi_q32[:count], np.uint32)
    if count == 0:
        idx = np.zeros(1, np.int32)
        pq = np.zeros(1, np.uint32)
    O = np.zeros((n_i, d), np.float64)
    lib().orc_ht_attention_block(Q, K, V, L, Lk, d, q_block, kv_block, i, idx, pq, int(count), O)
    return O


# ------------------------------------------------- many independent units

def run_units(fn, units, threads=None):
    """Run independent (single-threaded) oracle units on host threads.

    ctypes releases the GIL inside the C calls, so the units run in parallel.
    """
    threads = threads or os.cpu_count() or 1
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, units))

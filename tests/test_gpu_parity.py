"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

* ab_sample is bit-exact with the oracle's SIP on the same P (idx, pi_q32,
  count), including counter word 3 (b > 0) and capped rows.
* ab_attention on given lists (the oracle's or the GPU's) matches the oracle's
  reweighted attention within max-abs 2e-2 and relative L2 5e-3 (bf16 in and
  out, fp64 oracle); ab_attention_dense matches dense attention the same way.
* ab_select's P, from its own centroids, gives a selection that agrees with
  the oracle's (independent centroids) on >= 99.5% of kept blocks.
* Edge cases: ragged query and KV blocks, empty lists, full budget (then the
  sparse kernel equals the dense kernel bit for bit), every supported
  kv_block / q_block / d / C, bad lists reported as AB_ERR_CAPACITY.
"""
import numpy as np
import pytest

import oracle
from helpers import (assert_close_attention, np32, oracle_dense_units, oracle_ht_units, oracle_sip_rows,
                     rel_l2, selection_agreement)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_sparse_attention_queries_b200 as ab  # noqa: E402
from block_sparse_attention_queries_b200.synthetic import WORKLOADS, make_qkv, make_workload_qkv  # noqa: E402


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from block_sparse_attention_queries_b200 import build as abbuild
    abbuild.build()  # rebuilds only if a source is newer than libab.so
    ab.lib()  # the native library must load; there is no fallback
    return torch.device("cuda:0")


def _no_device_error(dev):
    code = ab.device_error(dev)
    assert code == 0, ab.status_string(code)


def _inputs(p, grid, F, seed, dev):
    Q, K, V = make_qkv(p.B, p.H, grid, p.d, F, seed=seed)
    return (Q, K, V), tuple(t.to(dev) for t in (Q, K, V)), tuple(np32(t) for t in (Q, K, V))


def _lists_np(idx, piq, cnt):
    return (idx.cpu().numpy(), piq.cpu().numpy().view(np.uint32), cnt.cpu().numpy())


def _all_units(p):
    return [(b, h, i) for b in range(p.B) for h in range(p.H) for i in range(p.Nq)]


def _stack_units(p, res, units):
    out = np.zeros((p.B, p.H, p.L, p.d))
    for (b, h, i) in units:
        o = res[(b, h, i)]
        out[b, h, i * p.q_block: i * p.q_block + o.shape[0]] = o
    return out


# ------------------------------------------------------------------ dense

@pytest.mark.parametrize("B,H,grid,d,qb", [(1, 1, (4, 16, 16), 64, 64), (2, 2, (3, 10, 10), 128, 128),
                                          (1, 2, (2, 7, 9), 64, 128), (1, 1, (1, 1, 5), 128, 64)])
def test_dense_matches_oracle(dev, B, H, grid, d, qb):
    L = grid[0] * grid[1] * grid[2]
    p = ab.Params(B=B, H=H, L=L, d=d, q_block=qb)
    _, (Q, K, V), (Qn, Kn, Vn) = _inputs(p, grid, 8, 7, dev)
    O = ab.ab_attention_dense(p, Q, K, V)
    torch.cuda.synchronize()
    _no_device_error(dev)
    ref = _stack_units(p, oracle_dense_units(Qn, Kn, Vn, qb, _all_units(p)), _all_units(p))
    assert_close_attention(np32(O), ref, "dense")


# ---------------------------------------------------------- sparse, given lists

def _oracle_lists(p, Qn, Kn, seed):
    """Oracle IBCS + SIP for every row: lists as numpy arrays of full capacity."""
    Kb = oracle.budget(p.Nkv, p.keep_ratio)
    P = np.zeros((p.B, p.H, p.Nq, p.Nkv), np.float32)
    for b in range(p.B):
        for h in range(p.H):
            P[b, h] = oracle.select_head(Qn[b, h], Kn[b, h], p.q_block, p.kv_block, p.C, p.kmeans_iters)
    idx, pq, cnt = oracle.sip(P, Kb, seed)
    return P, idx, pq, cnt


@pytest.mark.parametrize("name,d,qb,kvb,C,keep", [
    ("tiny", 64, 64, 16, 4, 0.10),
    ("ragged", 128, 128, 16, 8, 0.15),
    ("kv32", 128, 128, 32, 8, 0.20),
    ("kv64", 64, 128, 64, 4, 0.30),
    ("q64", 128, 64, 16, 2, 0.10),
])
def test_sparse_attention_on_oracle_lists(dev, name, d, qb, kvb, C, keep):
    grid = {"tiny": (4, 16, 16), "ragged": (3, 17, 19), "kv32": (4, 16, 20),
            "kv64": (5, 13, 11), "q64": (2, 16, 23)}[name]
    L = grid[0] * grid[1] * grid[2]
    p = ab.Params(B=1, H=2, L=L, d=d, q_block=qb, kv_block=kvb, C=C, keep_ratio=keep, seed=11)
    _, (Q, K, V), (Qn, Kn, Vn) = _inputs(p, grid, 8, 3, dev)
    _, idx, pq, cnt = _oracle_lists(p, Qn, Kn, p.seed)
    O = ab.ab_attention(p, Q, K, V, torch.from_numpy(idx).to(dev), torch.from_numpy(pq.view(np.int32)).to(dev),
                        torch.from_numpy(cnt).to(dev))
    torch.cuda.synchronize()
    _no_device_error(dev)
    units = _all_units(p)
    ref = _stack_units(p, oracle_ht_units(Qn, Kn, Vn, qb, kvb, units, idx, pq, cnt), units)
    assert_close_attention(np32(O), ref, name)


def test_empty_and_hand_made_lists(dev):
    # rows with count 0 give zeros; unsorted lists and arbitrary weights are accepted
    grid = (2, 8, 16)
    L = 256
    p = ab.Params(B=1, H=1, L=L, d=128, q_block=128, kv_block=16, C=4, keep_ratio=0.2)
    _, (Q, K, V), (Qn, Kn, Vn) = _inputs(p, grid, 8, 5, dev)
    idx = np.zeros((1, 1, 2, 16), np.int32)
    pq = np.zeros((1, 1, 2, 16), np.uint32)
    cnt = np.array([[[0, 11]]], np.int32)
    idx[0, 0, 1, :11] = [15, 3, 7, 0, 9, 1, 14, 2, 8, 12, 5]
    pq[0, 0, 1, :11] = [0, 123456789, 2**31, 4000000000, 1, 77, 0, 2**30, 999, 3**19, 2**32 - 1]
    O = ab.ab_attention(p, Q, K, V, torch.from_numpy(idx).to(dev), torch.from_numpy(pq.view(np.int32)).to(dev),
                        torch.from_numpy(cnt).to(dev))
    torch.cuda.synchronize()
    _no_device_error(dev)
    On = np32(O)
    assert not On[0, 0, :128].any()
    ref = oracle.ht_attention_block(Qn[0, 0], Kn[0, 0], Vn[0, 0], 128, 16, 1, idx[0, 0, 1], pq[0, 0, 1], 11)
    assert_close_attention(On[0, 0, 128:], ref, "hand-made")


def test_bad_lists_raise_capacity_without_fault(dev):
    p = ab.Params(B=1, H=1, L=256, d=64, q_block=128, kv_block=16, C=4, keep_ratio=0.2)
    _, (Q, K, V), _ = _inputs(p, (2, 8, 16), 8, 5, dev)
    idx = torch.zeros(1, 1, 2, 16, dtype=torch.int32, device=dev)
    piq = torch.zeros_like(idx)
    cnt = torch.tensor([[[3, 99]]], dtype=torch.int32, device=dev)   # count > Nkv
    idx[0, 0, 0, :3] = torch.tensor([1, 16, -2])                     # out of range entries
    ab.ab_attention(p, Q, K, V, idx, piq, cnt)
    torch.cuda.synchronize()
    assert ab.device_error(dev) == 4  # AB_ERR_CAPACITY
    assert ab.device_error(dev) == 0  # cleared by the read
    # a list whose every entry is invalid leaves no key: that block's output is
    # 0 (as for an empty list), not NaN; the other block is unaffected
    cnt2 = torch.tensor([[[2, 1]]], dtype=torch.int32, device=dev)
    idx2 = torch.zeros_like(idx)
    idx2[0, 0, 0, :2] = torch.tensor([16, -5])   # Nkv = 16: both out of range
    idx2[0, 0, 1, 0] = 3
    O = ab.ab_attention(p, Q, K, V, idx2, piq, cnt2)
    torch.cuda.synchronize()
    assert ab.device_error(dev) == 4
    O0 = O[0, 0, :128].float()
    assert torch.equal(O0, torch.zeros_like(O0))
    assert torch.isfinite(O[0, 0, 128:].float()).all()


def test_forward_slices_equal_forward(dev):
    # a layer's heads split into slices (as among GPUs), run one after the
    # other here: P, lists and output equal those heads of the whole-problem
    # call bit for bit (the draws use the whole problem's counters)
    p = ab.Params(B=2, H=3, L=1500, d=64, q_block=64, kv_block=16, C=4, keep_ratio=0.2, seed=5)
    _, (Q, K, V), _ = _inputs(p, (3, 20, 25), 8, 13, dev)
    full = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    Qf, Kf, Vf = (t.reshape(1, p.B * p.H, *t.shape[2:]) for t in (Q, K, V))
    for world in (2, 4):
        for bh0, nbh in ab.head_slices(p.B, p.H, world):
            sl = slice(bh0, bh0 + nbh)
            got = ab.ab_forward_slice(p, bh0, nbh, Qf[:, sl].contiguous(), Kf[:, sl].contiguous(),
                                      Vf[:, sl].contiguous())
            torch.cuda.synchronize()
            for name in ("P", "idx", "pi_q32", "count", "O"):
                a = getattr(full, name).reshape(p.B * p.H, *getattr(full, name).shape[2:])[sl]
                assert torch.equal(getattr(got, name)[0], a), (world, bh0, name)
    _no_device_error(dev)


# ------------------------------------------------------------------ sampler
# ------------------------------------------------------------------ sampler

def _skewed_P(B, H, Nq, Nkv, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, H, Nq, Nkv)) * rng.uniform(0.5, 6.0, (B, H, Nq, 1))
    P = np.exp(x - x.max(-1, keepdims=True))
    return (P / P.sum(-1, keepdims=True)).astype(np.float32)


def test_samplers_write_into_caller_buffers(dev):
    # out=(idx, pi_q32, count): the same lists as the allocating call, written in place
    p = ab.Params(B=1, H=2, L=3000, d=64, q_block=64, kv_block=16, C=4, keep_ratio=0.2, seed=11)
    P = torch.rand(p.B, p.H, p.Nq, p.Nkv, generator=torch.Generator().manual_seed(4)).to(dev)
    P = (P / P.sum(-1, keepdim=True)).contiguous()
    for fn in (ab.ab_sample, ab.ab_sample_systematic, ab.ab_sample_topk):
        ref = fn(p, P)
        out = (torch.full_like(ref[0], -7), torch.full_like(ref[1], -7), torch.full_like(ref[2], -7))
        got = fn(p, P, out=out)
        torch.cuda.synchronize()
        assert all(g.data_ptr() == o.data_ptr() for g, o in zip(got, out))
        assert torch.equal(got[2], ref[2])
        for r in range(p.Nq):
            c = int(ref[2][0, 0, r])
            assert torch.equal(got[0][0, 0, r, :c], ref[0][0, 0, r, :c])
            assert torch.equal(got[1][0, 0, r, :c], ref[1][0, 0, r, :c])
    _no_device_error(dev)


@pytest.mark.parametrize("B,H,L,kvb,keep,seed", [(2, 3, 1000, 16, 0.1, 42), (1, 2, 4096, 16, 0.5, 7),
                                                 (2, 1, 8192, 32, 0.05, 2**63 + 12345),
                                                 (1, 1, 2000, 64, 1.0, 3), (1, 2, 118800, 16, 0.08, 42),
                                                 (1, 1, 262400, 16, 0.02, 5)])
def test_sample_bit_exact(dev, B, H, L, kvb, keep, seed):
    # L = 262400 gives rows of 16400 KV blocks, longer than the sampler's
    # shared-memory row cache, so that case reads P from global memory.
    p = ab.Params(B=B, H=H, L=L, d=128, q_block=128, kv_block=kvb, C=8, keep_ratio=keep, seed=seed)
    Nq = min(p.Nq, 12) if L > 100000 else p.Nq
    P = _skewed_P(B, H, p.Nq, p.Nkv, seed % 1000)
    idx, piq, cnt = ab.ab_sample(p, torch.from_numpy(P).to(dev))
    torch.cuda.synchronize()
    _no_device_error(dev)
    gi, gp, gc = _lists_np(idx, piq, cnt)
    Kb = oracle.budget(p.Nkv, keep)
    assert Kb == ab.budget(p)
    rows = [(b, h, i) for b in range(B) for h in range(H) for i in range(Nq)]
    ref = oracle_sip_rows(P, Kb, seed, rows)
    for r in rows:
        oi, op, on = ref[r]
        assert gc[r] == on, r
        np.testing.assert_array_equal(gi[r][:on], oi)
        np.testing.assert_array_equal(gp[r][:on], op)


@pytest.mark.parametrize("B,H,L,kvb,keep,seed", [(2, 3, 1000, 16, 0.1, 42), (1, 2, 4096, 16, 0.5, 7),
                                                 (1, 1, 2000, 64, 1.0, 3), (1, 2, 118800, 16, 0.08, 42)])
def test_sample_topk_bit_exact(dev, B, H, L, kvb, keep, seed):
    # truncation (top-Kb, ties to the lower block, pi = 1) against the oracle,
    # with ties planted at each row's threshold
    p = ab.Params(B=B, H=H, L=L, d=128, q_block=128, kv_block=kvb, C=8, keep_ratio=keep, seed=seed)
    Nq = min(p.Nq, 12) if L > 100000 else p.Nq
    P = _skewed_P(B, H, p.Nq, p.Nkv, seed % 1000)
    Kb = oracle.budget(p.Nkv, keep)
    thr = np.sort(P, axis=-1)[..., -Kb]
    P[..., ::5] = thr[..., None]
    idx, piq, cnt = ab.ab_sample_topk(p, torch.from_numpy(P).to(dev))
    torch.cuda.synchronize()
    _no_device_error(dev)
    gi, gp, gc = _lists_np(idx, piq, cnt)
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                oi, op, on = oracle.topk_row(P[b, h, i], Kb)
                assert gc[b, h, i] == on == Kb
                np.testing.assert_array_equal(gi[b, h, i, :on], oi)
                np.testing.assert_array_equal(gp[b, h, i, :on], op)


def test_truncated_attention_small_workload(dev):
    # the whole truncation path: ab_select -> ab_sample_topk -> ab_attention
    w = WORKLOADS["small"]
    p = ab.Params.of(w)
    Qc, Kc, Vc = make_workload_qkv(w)
    Q, K, V = (t.to(dev) for t in (Qc, Kc, Vc))
    P = ab.ab_select(p, Q, K)
    idx, piq, cnt = ab.ab_sample_topk(p, P)
    O = ab.ab_attention(p, Q, K, V, idx, piq, cnt)
    torch.cuda.synchronize()
    _no_device_error(dev)
    gi, gp, gc = _lists_np(idx, piq, cnt)
    Kb = oracle.budget(p.Nkv, p.keep_ratio)
    Pg = P.cpu().numpy()
    units = _all_units(p)
    for (b, h, i) in units[::7]:
        oi, _, _ = oracle.topk_row(Pg[b, h, i], Kb)
        np.testing.assert_array_equal(gi[b, h, i, :Kb], oi)
    Qn, Kn, Vn = np32(Qc), np32(Kc), np32(Vc)
    ref = _stack_units(p, oracle_ht_units(Qn, Kn, Vn, p.q_block, p.kv_block, units, gi, gp, gc), units)
    assert_close_attention(np32(O), ref, "truncated small")


@pytest.mark.parametrize("B,H,L,kvb,keep,seed", [(2, 3, 1000, 16, 0.1, 42), (1, 2, 4096, 16, 0.5, 7),
                                                 (2, 1, 8192, 32, 0.05, 2**63 + 12345),
                                                 (1, 1, 2000, 64, 1.0, 3), (1, 2, 32760, 16, 0.11, 9),
                                                 (1, 2, 118800, 16, 0.08, 42), (1, 1, 262400, 16, 0.02, 5)])
def test_sample_systematic_bit_exact(dev, B, H, L, kvb, keep, seed):
    p = ab.Params(B=B, H=H, L=L, d=128, q_block=128, kv_block=kvb, C=8, keep_ratio=keep, seed=seed)
    Nq = min(p.Nq, 12) if L > 100000 else p.Nq
    P = _skewed_P(B, H, p.Nq, p.Nkv, seed % 1000)
    idx, piq, cnt = ab.ab_sample_systematic(p, torch.from_numpy(P).to(dev))
    torch.cuda.synchronize()
    _no_device_error(dev)
    gi, gp, gc = _lists_np(idx, piq, cnt)
    Kb = oracle.budget(p.Nkv, keep)
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                oi, op, on = oracle.systematic_row(P[b, h, i], Kb, seed, b, h, i)
                assert gc[b, h, i] == on and Kb - 1 <= on <= Kb
                np.testing.assert_array_equal(gi[b, h, i, :on], oi)
                np.testing.assert_array_equal(gp[b, h, i, :on], op)


def test_systematic_attention_small_workload(dev):
    # ab_select -> ab_sample_systematic -> ab_attention against the oracle
    w = WORKLOADS["small"]
    p = ab.Params.of(w)
    Qc, Kc, Vc = make_workload_qkv(w)
    Q, K, V = (t.to(dev) for t in (Qc, Kc, Vc))
    P = ab.ab_select(p, Q, K)
    idx, piq, cnt = ab.ab_sample_systematic(p, P)
    O = ab.ab_attention(p, Q, K, V, idx, piq, cnt)
    torch.cuda.synchronize()
    _no_device_error(dev)
    gi, gp, gc = _lists_np(idx, piq, cnt)
    units = _all_units(p)
    Qn, Kn, Vn = np32(Qc), np32(Kc), np32(Vc)
    ref = _stack_units(p, oracle_ht_units(Qn, Kn, Vn, p.q_block, p.kv_block, units, gi, gp, gc), units)
    assert_close_attention(np32(O), ref, "systematic small")


def test_philox_word3_matches_curand_device():
    # cuRAND's device Philox4x32_10 (a library routine) vs the oracle on
    # counters with all four words populated.
    import ctypes
    import os
    import subprocess
    here = os.path.dirname(os.path.abspath(__file__))
    so = os.path.join(here, "cuda", "curand_philox.so")
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared", "-Xcompiler",
                           "-fPIC", "-o", so, os.path.join(here, "cuda", "curand_philox.cu")])
    lib = ctypes.CDLL(so)
    rng = np.random.default_rng(0)
    n = 4096
    ctr = rng.integers(0, 2**32, (n, 4), dtype=np.uint64).astype(np.uint32)
    key = rng.integers(0, 2**32, (n, 2), dtype=np.uint64).astype(np.uint32)
    out = np.zeros((n, 4), np.uint32)
    assert lib.curand_philox_many(ctr.ctypes.data_as(ctypes.c_void_p), key.ctypes.data_as(ctypes.c_void_p),
                                  out.ctypes.data_as(ctypes.c_void_p), n) == 0
    for k in range(n):
        np.testing.assert_array_equal(oracle.philox4x32_10(ctr[k], key[k]), out[k])


# ------------------------------------------------------------------ selector

@pytest.mark.parametrize("wname,C", [("tiny", 4), ("small", 8), ("small", 16), ("small", 1)])
def test_select_agrees_with_oracle(dev, wname, C):
    w = WORKLOADS[wname].with_(C=C)
    p = ab.Params.of(w)
    Qc, Kc, Vc = make_workload_qkv(w)
    Q, K = Qc.to(dev), Kc.to(dev)
    P, cent, cnts = ab.ab_select(p, Q, K, want_centroids=True)
    torch.cuda.synchronize()
    _no_device_error(dev)
    Pg = P.cpu().numpy()
    np.testing.assert_allclose(Pg.sum(-1), 1.0, atol=2e-4)
    Qn, Kn = np32(Qc), np32(Kc)
    Po = np.zeros_like(Pg)
    for b in range(p.B):
        for h in range(p.H):
            Po[b, h] = oracle.select_head(Qn[b, h], Kn[b, h], p.q_block, p.kv_block, C, p.kmeans_iters)
    # block-mass estimates agree closely
    assert rel_l2(Pg, Po) < 2e-2, rel_l2(Pg, Po)
    # selection from GPU P vs selection from the oracle's own P, same seed
    Kb = oracle.budget(p.Nkv, p.keep_ratio)
    rows = _all_units(p)
    so = oracle_sip_rows(Po, Kb, p.seed, rows)
    idx, piq, cnt = ab.ab_sample(p, P)
    gi, gp, gc = _lists_np(idx, piq, cnt)
    selection_agreement([(gi[r][:gc[r]], so[r][0]) for r in rows], f"{wname} C={C}")
    # the sampler is bit-exact on the GPU's own P
    sg = oracle_sip_rows(Pg, Kb, p.seed, rows)
    for r in rows:
        assert gc[r] == sg[r][2]
        np.testing.assert_array_equal(gi[r][:gc[r]], sg[r][0])
        np.testing.assert_array_equal(gp[r][:gc[r]], sg[r][1])


def test_kmeans_centroids_close_to_oracle(dev):
    w = WORKLOADS["small"]
    p = ab.Params.of(w)
    Qc, Kc, _ = make_workload_qkv(w)
    _, cent, cnts = ab.ab_select(p, Qc.to(dev), Kc.to(dev), want_centroids=True)
    torch.cuda.synchronize()
    cent, cnts = cent.cpu().numpy(), cnts.cpu().numpy()
    Qn, Kn = np32(Qc), np32(Kc)
    same = 0
    for h in range(p.H):
        _, mu, cn = oracle.select_head(Qn[0, h], Kn[0, h], p.q_block, p.kv_block, p.C, p.kmeans_iters,
                                       want_centroids=True)
        for i in range(p.Nq):
            if (cn[i] == cnts[0, h, i]).all():
                same += 1
                np.testing.assert_allclose(cent[0, h, i], mu[i], rtol=0, atol=1e-4)
    assert same >= 0.9 * p.H * p.Nq


# ------------------------------------------------------------- whole path

def test_small_workload_end_to_end(dev):
    w = WORKLOADS["small"]
    p = ab.Params.of(w)
    Qc, Kc, Vc = make_workload_qkv(w)
    Q, K, V = (t.to(dev) for t in (Qc, Kc, Vc))
    bufs = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    _no_device_error(dev)
    Qn, Kn, Vn = np32(Qc), np32(Kc), np32(Vc)
    gi, gp, gc = _lists_np(bufs.idx, bufs.pi_q32, bufs.count)
    units = _all_units(p)
    ref = _stack_units(p, oracle_ht_units(Qn, Kn, Vn, p.q_block, p.kv_block, units, gi, gp, gc), units)
    assert_close_attention(np32(bufs.O), ref, "small")
    # and the sampler on the GPU's P is bit-exact
    Kb = oracle.budget(p.Nkv, p.keep_ratio)
    sg = oracle_sip_rows(bufs.P.cpu().numpy(), Kb, p.seed, units)
    for r in units:
        assert gc[r] == sg[r][2]
        np.testing.assert_array_equal(gi[r][:gc[r]], sg[r][0])


@pytest.mark.parametrize("L,qb,kvb,C", [(1, 64, 16, 1), (5, 128, 16, 4), (17, 64, 16, 16), (130, 128, 64, 2),
                                         (257, 128, 32, 8)])
def test_tiny_sequences_end_to_end(dev, L, qb, kvb, C):
    # degenerate sizes: a single token, one partial KV block, fewer queries
    # than clusters, a ragged last query block of 1-2 rows
    p = ab.Params(B=1, H=2, L=L, d=64, q_block=qb, kv_block=kvb, C=C, keep_ratio=0.3, seed=5)
    grid = (1, 1, L)
    (Qc, Kc, Vc), (Q, K, V), (Qn, Kn, Vn) = _inputs(p, grid, 8, 21, dev)
    bufs = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    _no_device_error(dev)
    gi, gp, gc = _lists_np(bufs.idx, bufs.pi_q32, bufs.count)
    Kb = oracle.budget(p.Nkv, p.keep_ratio)
    units = _all_units(p)
    sg = oracle_sip_rows(bufs.P.cpu().numpy(), Kb, p.seed, units)
    for r in units:
        assert gc[r] == sg[r][2]
        np.testing.assert_array_equal(gi[r][:gc[r]], sg[r][0])
    ref = _stack_units(p, oracle_ht_units(Qn, Kn, Vn, p.q_block, p.kv_block, units, gi, gp, gc), units)
    assert_close_attention(np32(bufs.O), ref, f"tiny L={L}")
    Od = ab.ab_attention_dense(p, Q, K, V)
    torch.cuda.synchronize()
    refd = _stack_units(p, oracle_dense_units(Qn, Kn, Vn, p.q_block, units), units)
    assert_close_attention(np32(Od), refd, f"tiny dense L={L}")


@pytest.mark.parametrize("B,H,grid", [(2, 3, (2, 16, 16)), (1, 9, (2, 12, 20)), (1, 2, (2, 16, 16))])
def test_forward_host_equals_device_path(dev, B, H, grid):
    # ab_forward_host (pinned host buffers in and out; head groups pipelined
    # over PCIe when B*H > 4) gives the device path's lists and output bit for bit
    L = grid[0] * grid[1] * grid[2]
    p = ab.Params(B=B, H=H, L=L, d=128, q_block=128, kv_block=16, C=8, keep_ratio=0.15, seed=99)
    (Qc, Kc, Vc), (Q, K, V), _ = _inputs(p, grid, 8, 13, dev)
    ref = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    Qh, Kh, Vh = (t.pin_memory() for t in (Qc, Kc, Vc))
    Oh = torch.empty_like(Qc).pin_memory()
    Qd, Kd, Vd = (torch.empty_like(t) for t in (Q, K, V))
    bufs = ab.Buffers(p, dev)
    ab.ab_forward_host(p, Qh, Kh, Vh, Oh, Qd, Kd, Vd, bufs, dev)
    torch.cuda.synchronize()
    _no_device_error(dev)
    assert torch.equal(bufs.count, ref.count)
    assert torch.equal(bufs.idx, ref.idx)
    assert torch.equal(bufs.pi_q32, ref.pi_q32)
    assert torch.equal(bufs.O, ref.O)
    assert torch.equal(Oh, ref.O.cpu())


def test_forward_captured_in_cuda_graph(dev):
    # the whole path captured into a CUDA graph (the selector's side stream
    # joins the capture through its fork and join events) and replayed gives
    # the eager call's lists and output bit for bit, replay after replay
    grid = (2, 16, 16)
    p = ab.Params(B=1, H=3, L=512, d=128, q_block=128, kv_block=16, C=8, keep_ratio=0.15, seed=17)
    _, (Q, K, V), _ = _inputs(p, grid, 8, 23, dev)
    ref = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    bufs = ab.Buffers(p, dev)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        ab.ab_forward(p, Q, K, V, bufs)  # first call on this stream outside the capture
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ab.ab_forward(p, Q, K, V, bufs)
    for _ in range(3):
        bufs.O.zero_()
        bufs.count.zero_()
        g.replay()
        torch.cuda.synchronize()
        _no_device_error(dev)
        assert torch.equal(bufs.count, ref.count)
        assert torch.equal(bufs.idx, ref.idx)
        assert torch.equal(bufs.O, ref.O)


def test_forward_host_repeated_and_from_two_threads(dev):
    # the pipelined host call keeps its copy streams and events per CUDA
    # context: repeated calls, and calls from two host threads at once (each
    # on its own stream with its own buffers), all give ab_forward's results
    import threading
    grid = (2, 16, 16)
    p = ab.Params(B=1, H=9, L=512, d=128, q_block=128, kv_block=16, C=8, keep_ratio=0.15, seed=5)
    (Qc, Kc, Vc), (Q, K, V), _ = _inputs(p, grid, 8, 21, dev)
    ref = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    results, errors = {}, []

    def worker(k):
        try:
            st = torch.cuda.Stream(dev)
            with torch.cuda.stream(st):
                Qh, Kh, Vh = (t.pin_memory() for t in (Qc, Kc, Vc))
                Oh = torch.empty_like(Qc).pin_memory()
                Qd, Kd, Vd = (torch.empty_like(t) for t in (Q, K, V))
                bufs = ab.Buffers(p, dev)
                Oh.zero_()
                for _ in range(3):
                    ab.ab_forward_host(p, Qh, Kh, Vh, Oh, Qd, Kd, Vd, bufs, dev)
                st.synchronize()
                res = (Oh.clone(), bufs.idx.clone(), bufs.count.clone())
                st.synchronize()
                results[k] = res
        except Exception as e:  # reported below, on the main thread
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(k,)) for k in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    _no_device_error(dev)
    for k in range(2):
        Oh, idx, cnt = results[k]
        assert torch.equal(cnt, ref.count)
        assert torch.equal(idx, ref.idx)
        assert torch.equal(Oh, ref.O.cpu())


@pytest.mark.parametrize("d,kvb", [(128, 16), (64, 32), (128, 64)])
def test_full_budget_equals_dense_bitwise(dev, d, kvb):
    grid = (4, 18, 20)  # L = 1440: ragged last query block and last KV block for 64
    L = 1440
    p = ab.Params(B=1, H=2, L=L, d=d, q_block=128, kv_block=kvb, C=4, keep_ratio=1.0)
    _, (Q, K, V), _ = _inputs(p, grid, 8, 9, dev)
    bufs = ab.ab_forward(p, Q, K, V)
    Od = ab.ab_attention_dense(p, Q, K, V)
    torch.cuda.synchronize()
    _no_device_error(dev)
    assert (bufs.count == p.Nkv).all()
    assert (bufs.pi_q32 == 0).all()
    assert torch.equal(bufs.O, Od)

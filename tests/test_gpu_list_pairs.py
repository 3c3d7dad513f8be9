"""Sparse attention on hand-made lists for the two query blocks that one CTA
computes (AB-Attention page, "AB-Attention ve Üç Temel Yeniliği",
hardware-friendly kernel and SIP items: each query block's output is its own
1/pi-weighted attention over its own list): identical lists, one list inside
the other, disjoint lists, lists with few common blocks, ragged counts,
repeated entries (a block listed twice counts twice, as in the oracle),
lists out of order, and out-of-range entries at the ends of ascending lists
(skipped, with the capacity error).  Each output block is compared with the
oracle's reweighted attention over that block's list."""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import oracle  # noqa: E402
from helpers import assert_close_attention, np32  # noqa: E402

torch = pytest.importorskip("torch")

import block_sparse_attention_queries_b200 as ab  # noqa: E402
from block_sparse_attention_queries_b200.synthetic import make_qkv  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda:0")


def _pair_lists(kind, Nkv, rng):
    """Two block lists (query blocks 2k, 2k+1) of the given kind."""
    def pick(n):
        return np.sort(rng.choice(Nkv, size=min(n, Nkv), replace=False))
    if kind == "same":
        a = pick(rng.integers(8, Nkv))
        return a, a.copy()
    if kind == "subset":
        a = pick(rng.integers(16, Nkv))
        b = np.sort(rng.choice(a, size=len(a) // 2 + 3, replace=False))
        return a, b
    if kind == "disjoint":
        perm = rng.permutation(Nkv)
        n = Nkv // 3
        return np.sort(perm[:n]), np.sort(perm[n:2 * n + 5])
    if kind == "few":  # fewer common blocks than slots in a tile
        perm = rng.permutation(Nkv)
        a, b = np.sort(perm[:40]), np.sort(np.concatenate([perm[40:70], perm[:3]]))
        return a, b
    if kind == "overlap":
        a = pick(rng.integers(8, max(9, Nkv // 2)))
        extra = pick(rng.integers(4, max(5, Nkv // 2)))
        keep = a[rng.random(len(a)) < 0.4]
        return a, np.unique(np.concatenate([keep, extra]))
    if kind == "unsorted":
        a = pick(60)
        b = a.copy()
        b[[3, 4]] = b[[4, 3]]
        return a, b
    if kind == "dup":
        a = pick(50)
        b = np.sort(np.concatenate([a[:30], a[5:7]]))
        return a, b
    raise ValueError(kind)


@pytest.mark.parametrize("kvb,d,grid", [(16, 128, (4, 16, 64)), (32, 128, (4, 16, 64)), (64, 64, (3, 16, 52)),
                                        (16, 64, (2, 30, 33))])
def test_list_pairs_match_oracle(dev, kvb, d, grid):
    L = grid[0] * grid[1] * grid[2]
    p = ab.Params(B=1, H=2, L=L, d=d, q_block=128, kv_block=kvb, C=4, keep_ratio=0.2, seed=3)
    Qc, Kc, Vc = make_qkv(p.B, p.H, grid, p.d, 8, seed=9)
    Q, K, V = (t.to(dev) for t in (Qc, Kc, Vc))
    Qn, Kn, Vn = np32(Qc), np32(Kc), np32(Vc)
    rng = np.random.default_rng(kvb * 1000 + d)
    kinds = ["same", "subset", "disjoint", "few", "overlap", "unsorted", "dup", "overlap"]
    idx = np.zeros((p.B, p.H, p.Nq, p.Nkv), np.int32)
    pq = np.zeros((p.B, p.H, p.Nq, p.Nkv), np.uint32)
    cnt = np.zeros((p.B, p.H, p.Nq), np.int32)
    for h in range(p.H):
        for k in range(p.Nq // 2):
            a, b = _pair_lists(kinds[(k + 3 * h) % len(kinds)], p.Nkv, rng)
            for s, lst in enumerate((a, b)):
                i = 2 * k + s
                cnt[0, h, i] = len(lst)
                idx[0, h, i, :len(lst)] = lst
                w = rng.integers(1, 2**32, size=len(lst), dtype=np.uint64).astype(np.uint32)
                w[rng.random(len(lst)) < 0.2] = 0  # Pi = 1
                pq[0, h, i, :len(lst)] = w
        if p.Nq % 2:
            i = p.Nq - 1
            lst = np.sort(rng.choice(p.Nkv, size=17, replace=False))
            cnt[0, h, i] = 17
            idx[0, h, i, :17] = lst
    O = ab.ab_attention(p, Q, K, V, torch.from_numpy(idx).to(dev), torch.from_numpy(pq.view(np.int32)).to(dev),
                        torch.from_numpy(cnt).to(dev))
    torch.cuda.synchronize()
    assert ab.device_error(dev) == 0
    On = np32(O)
    units = [(h, i) for h in range(p.H) for i in range(p.Nq)]

    def one(u):
        h, i = u
        return u, oracle.ht_attention_block(Qn[0, h], Kn[0, h], Vn[0, h], p.q_block, kvb, i, idx[0, h, i],
                                            pq[0, h, i], int(cnt[0, h, i]))
    for (h, i), ref in oracle.run_units(one, units):
        got = On[0, h, i * p.q_block: i * p.q_block + ref.shape[0]]
        assert_close_attention(got, ref, f"h={h} block {i}")


def test_list_pairs_with_out_of_range_ends(dev):
    # ascending lists with an invalid entry at each end: those are skipped
    # (capacity error) and each output is the attention over the list's valid
    # entries
    grid = (4, 16, 32)
    L = 2048
    p = ab.Params(B=1, H=1, L=L, d=128, q_block=128, kv_block=16, C=4, keep_ratio=0.2)
    Qc, Kc, Vc = make_qkv(1, 1, grid, 128, 8, seed=4)
    Q, K, V = (t.to(dev) for t in (Qc, Kc, Vc))
    Qn, Kn, Vn = np32(Qc), np32(Kc), np32(Vc)
    rng = np.random.default_rng(5)
    common = np.sort(rng.choice(np.arange(1, p.Nkv - 1), size=40, replace=False))
    a = np.concatenate([[-4], common, [p.Nkv + 1]]).astype(np.int32)
    b = np.concatenate([[-1], common[::2], [p.Nkv]]).astype(np.int32)
    idx = np.zeros((1, 1, p.Nq, p.Nkv), np.int32)
    pq = np.zeros((1, 1, p.Nq, p.Nkv), np.uint32)
    cnt = np.zeros((1, 1, p.Nq), np.int32)
    for i, lst in enumerate((a, b)):
        idx[0, 0, i, :len(lst)] = lst
        pq[0, 0, i, :len(lst)] = rng.integers(1, 2**32, size=len(lst), dtype=np.uint64).astype(np.uint32)
        cnt[0, 0, i] = len(lst)
    O = ab.ab_attention(p, Q, K, V, torch.from_numpy(idx).to(dev), torch.from_numpy(pq.view(np.int32)).to(dev),
                        torch.from_numpy(cnt).to(dev))
    torch.cuda.synchronize()
    assert ab.device_error(dev) == 4  # AB_ERR_CAPACITY, read and cleared
    On = np32(O)
    for i in range(2):
        keep = (idx[0, 0, i, :cnt[0, 0, i]] >= 0) & (idx[0, 0, i, :cnt[0, 0, i]] < p.Nkv)
        li, lp = idx[0, 0, i, :cnt[0, 0, i]][keep], pq[0, 0, i, :cnt[0, 0, i]][keep]
        ref = oracle.ht_attention_block(Qn[0, 0], Kn[0, 0], Vn[0, 0], 128, 16, i, li, lp, len(li))
        assert_close_attention(On[0, 0, i * 128:(i + 1) * 128], ref, f"block {i}")

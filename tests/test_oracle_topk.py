"""Pins of the oracle's truncation selection (top-Kb, pi = 1).

AB-Attention page: truncation drops the pruned blocks from the softmax
entirely (section "Video Difüzyon Modellerinde Dikkat (Attention)
Darboğazı"); SIP replaces it (section "AB-Attention ve Üç Temel Yeniliği").
Reading: the Kb blocks with the largest P, ties to the lower j, ascending,
no reweighting.  Pinned against numpy's stable sort (a library routine),
order invariants, special cases, and torch SDPA over the kept keys."""
import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")


def _library_topk(P, Kb):
    order = np.argsort(-P.astype(np.float64), kind="stable")  # descending, ties in index order
    return np.sort(order[:Kb]).astype(np.int32)


@pytest.mark.parametrize("Nkv,Kb,seed", [(64, 6, 0), (512, 51, 1), (2048, 225, 2), (7425, 594, 3), (33, 33, 4)])
def test_topk_matches_numpy_stable_sort(Nkv, Kb, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(Nkv) * 3
    P = np.exp(x - x.max())
    P = (P / P.sum()).astype(np.float32)
    # plant ties around the threshold
    P[::7] = np.sort(P)[-Kb] if Kb < Nkv else P[::7]
    idx, pq, n = oracle.topk_row(P, Kb)
    assert n == Kb
    np.testing.assert_array_equal(idx, _library_topk(P, Kb))
    assert not pq.any()


def test_topk_invariants_and_ties():
    rng = np.random.default_rng(7)
    P = rng.integers(0, 5, 300).astype(np.float32) / 10.0  # many ties
    Kb = 77
    idx, _, n = oracle.topk_row(P, Kb)
    kept = np.zeros(300, bool)
    kept[idx] = True
    assert n == Kb and np.all(np.diff(idx) > 0)
    assert P[kept].min() >= P[~kept].max()
    t = P[kept].min()
    tie_kept = np.nonzero(kept & (P == t))[0]
    tie_dropped = np.nonzero(~kept & (P == t))[0]
    if len(tie_dropped):
        assert tie_kept.max() < tie_dropped.min()  # ties go to the lower j


def test_topk_special_cases():
    P = np.full(50, 0.02, np.float32)
    np.testing.assert_array_equal(oracle.topk_row(P, 10)[0], np.arange(10))   # uniform: the first Kb
    np.testing.assert_array_equal(oracle.topk_row(P, 50)[0], np.arange(50))   # Kb = Nkv: all
    P2 = np.full(50, 0.001, np.float32)
    P2[37] = 0.9
    np.testing.assert_array_equal(oracle.topk_row(P2, 1)[0], [37])            # the dominant block


def test_truncated_attention_is_dense_attention_over_kept_blocks():
    rng = np.random.default_rng(11)
    L, d, qb, kvb = 200, 64, 64, 16
    Q = rng.standard_normal((L, d)).astype(np.float32)
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = rng.standard_normal((L, d)).astype(np.float32)
    Nkv = -(-L // kvb)
    P = rng.random(Nkv).astype(np.float32)
    idx, pq, n = oracle.topk_row(P, 5)
    i = 1
    O = oracle.ht_attention_block(Q, K, V, qb, kvb, i, idx, pq, n)
    keys = np.concatenate([np.arange(j * kvb, min(L, (j + 1) * kvb)) for j in idx])
    q = torch.from_numpy(Q[i * qb:(i + 1) * qb]).double()[None, None]
    k = torch.from_numpy(K[keys]).double()[None, None]
    v = torch.from_numpy(V[keys]).double()[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v)[0, 0].numpy()
    np.testing.assert_allclose(O, ref, rtol=1e-10, atol=1e-12)

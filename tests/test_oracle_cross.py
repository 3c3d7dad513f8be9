"""Pins for the oracle with queries and keys from sequences of different
lengths (Cross-Attention glossary page, "Cross-Attention Nasıl Çalışır?": the
queries come from one sequence, the keys and values from another; the kernel
softmax(QK^T/sqrt(d))V is the same).

Query blocks follow the query length L, KV blocks the key length Lk:

* dense attention with L != Lk equals torch's scaled_dot_product_attention in
  float64 (a library routine the oracle does not call);
* the reweighted block attention with every KV block kept at pi = 1 equals it
  too, with a ragged last query block and a ragged last KV block;
* a subset of KV blocks attends to exactly those keys, never to keys beyond Lk;
* IBCS closed forms with L != Lk: one cluster and one key per KV block gives
  scipy's softmax_j(mean query . k_j / sqrt(d)); identical keys give
  P_j = n_j / Lk.
"""
import numpy as np
import pytest
import torch
from scipy.special import softmax

import oracle


def _sdpa64(q, K, V):
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(K), t(V))[0, 0].numpy()


def _cross(L, Lk, d, seed):
    rng = np.random.default_rng(seed)
    Q = (rng.standard_normal((L, d)) * 1.5).astype(np.float32)
    K = rng.standard_normal((Lk, d)).astype(np.float32)
    V = rng.standard_normal((Lk, d)).astype(np.float32)
    return Q, K, V


@pytest.mark.parametrize("L,Lk,d", [(37, 90, 16), (130, 20, 64), (1, 300, 32), (200, 1, 16)])
def test_dense_cross_matches_sdpa(L, Lk, d):
    Q, K, V = _cross(L, Lk, d, L * 7 + Lk)
    np.testing.assert_allclose(oracle.dense_rows(Q, K, V), _sdpa64(Q, K, V), rtol=1e-12, atol=1e-12)
    part = oracle.dense_rows(Q, K, V, row0=L - 1, nrows=1)
    np.testing.assert_allclose(part, _sdpa64(Q[L - 1:], K, V), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("L,Lk,d,qb,kb", [(100, 70, 16, 64, 16), (70, 200, 32, 64, 32),
                                          (150, 131, 64, 128, 64)])
def test_full_list_with_unit_pi_is_dense_cross(L, Lk, d, qb, kb):
    Q, K, V = _cross(L, Lk, d, L + Lk + d)
    Nkv = -(-Lk // kb)
    idx = np.arange(Nkv, dtype=np.int32)
    pq = np.zeros(Nkv, np.uint32)
    ref = _sdpa64(Q, K, V)
    for i in range(-(-L // qb)):
        O = oracle.ht_attention_block(Q, K, V, qb, kb, i, idx, pq, Nkv)
        assert O.shape[0] == min(qb, L - i * qb)
        np.testing.assert_allclose(O, ref[i * qb: i * qb + O.shape[0]], rtol=1e-11, atol=1e-12)


def test_subset_attends_to_its_keys_only_ragged_key_sequence():
    L, Lk, d, qb, kb = 200, 38, 16, 64, 16          # Lk: blocks of 16, 16 and 6 keys
    Q, K, V = _cross(L, Lk, d, 5)
    sel = np.array([0, 2], np.int32)
    pq = np.zeros(2, np.uint32)
    keys = np.r_[0:16, 32:38]
    for i in range(-(-L // qb)):
        O = oracle.ht_attention_block(Q, K, V, qb, kb, i, sel, pq, 2)
        np.testing.assert_allclose(O, _sdpa64(Q[i * qb: min(L, (i + 1) * qb)], K[keys], V[keys]),
                                   rtol=1e-11, atol=1e-12)


def test_block_mass_cross_c1_bk1_is_softmax_of_mean_query():
    rng = np.random.default_rng(17)
    L, Lk, d = 40, 75, 16
    Q = rng.standard_normal((L, d)).astype(np.float32)
    K = rng.standard_normal((Lk, d)).astype(np.float32)
    P = oracle.select_head(Q, K, q_block=64, kv_block=1, C=1, iters=3)
    assert P.shape == (1, Lk)
    qbar = Q.astype(np.float64).mean(0)
    np.testing.assert_allclose(P[0], softmax(K.astype(np.float64) @ qbar / np.sqrt(d)), rtol=1e-12)


@pytest.mark.parametrize("L,Lk", [(100, 45), (30, 170)])
def test_block_mass_cross_equal_keys_is_block_share(L, Lk):
    rng = np.random.default_rng(L + Lk)
    d, qb, kb = 8, 32, 16
    Q = rng.standard_normal((L, d)).astype(np.float32)
    K = np.tile(rng.standard_normal((1, d)).astype(np.float32), (Lk, 1))
    P = oracle.select_head(Q, K, q_block=qb, kv_block=kb, C=4, iters=3)
    assert P.shape == (-(-L // qb), -(-Lk // kb))
    n_j = np.array([min(kb, Lk - j * kb) for j in range(-(-Lk // kb))], np.float64)
    for row in P:
        np.testing.assert_allclose(row, n_j / Lk, rtol=1e-12)


def test_select_head_cross_rows_follow_the_query_sequence():
    rng = np.random.default_rng(19)
    L, Lk, d = 150, 64, 16
    Q = rng.standard_normal((L, d)).astype(np.float32)
    K = rng.standard_normal((Lk, d)).astype(np.float32)
    P, mu, cnt = oracle.select_head(Q, K, 64, 16, 4, 3, want_centroids=True)
    assert P.shape == (3, 4)
    # the last query block has L - 128 = 22 queries; its centroids are the
    # k-means of exactly those rows
    assert cnt[2].sum() == 22
    mu2, cnt2 = oracle.kmeans(Q[128:], 4, 3)
    np.testing.assert_array_equal(mu[2], mu2)
    np.testing.assert_array_equal(cnt[2], cnt2)
    np.testing.assert_allclose(P.sum(1), 1.0, atol=1e-12)

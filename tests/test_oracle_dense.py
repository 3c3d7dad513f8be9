"""Pins for the oracle's dense attention softmax(QK^T/sqrt(d))V (Cross-Attention
glossary page, "Cross-Attention Nasıl Çalışır?").

Pinned against torch's scaled_dot_product_attention in float64 (a library
routine, not called by the oracle) and against closed forms.
"""
import numpy as np
import pytest
import torch

import oracle


def _sdpa64(Q, K, V):
    q = torch.from_numpy(np.asarray(Q, np.float64))[None, None]
    k = torch.from_numpy(np.asarray(K, np.float64))[None, None]
    v = torch.from_numpy(np.asarray(V, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v)[0, 0].numpy()


@pytest.mark.parametrize("L,d", [(1, 8), (37, 16), (130, 64), (77, 128)])
def test_dense_matches_sdpa_fp64(L, d):
    rng = np.random.default_rng(L * 1000 + d)
    Q = rng.standard_normal((L, d)).astype(np.float32) * 2
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = rng.standard_normal((L, d)).astype(np.float32)
    O = oracle.dense_rows(Q, K, V)
    np.testing.assert_allclose(O, _sdpa64(Q, K, V), rtol=1e-12, atol=1e-12)


def test_dense_row_window():
    rng = np.random.default_rng(3)
    Q, K, V = (rng.standard_normal((50, 16)).astype(np.float32) for _ in range(3))
    full = oracle.dense_rows(Q, K, V)
    part = oracle.dense_rows(Q, K, V, row0=13, nrows=9)
    np.testing.assert_array_equal(full[13:22], part)


def test_dense_zero_query_is_mean_of_values():
    rng = np.random.default_rng(4)
    L, d = 45, 32
    Q = np.zeros((L, d), np.float32)
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = rng.standard_normal((L, d)).astype(np.float32)
    O = oracle.dense_rows(Q, K, V)
    np.testing.assert_allclose(O, np.tile(V.astype(np.float64).mean(0), (L, 1)), rtol=1e-13, atol=1e-13)


def test_dense_one_hot_values_give_probability_rows():
    # V = identity (L = d): O is the attention matrix itself, rows sum to one.
    rng = np.random.default_rng(5)
    L = d = 24
    Q = rng.standard_normal((L, d)).astype(np.float32)
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = np.eye(L, dtype=np.float32)
    A = oracle.dense_rows(Q, K, V)
    assert (A > 0).all()
    np.testing.assert_allclose(A.sum(1), 1.0, rtol=0, atol=1e-14)


def test_dense_key_shift_invariance_and_permutation_equivariance():
    rng = np.random.default_rng(6)
    L, d = 40, 16
    Q, K, V = (rng.standard_normal((L, d)).astype(np.float32) for _ in range(3))
    K = (np.round(K * 64) / 64).astype(np.float32)  # so that K + u is exact in fp32
    O = oracle.dense_rows(Q, K, V)
    # adding one vector to every key adds a per-query constant to its logits
    u = np.float32(0.25) * np.ones(d, np.float32)
    O2 = oracle.dense_rows(Q, K + u, V)
    np.testing.assert_allclose(O, O2, rtol=1e-9, atol=1e-9)
    # permuting keys and values together does not change the output
    perm = rng.permutation(L)
    O3 = oracle.dense_rows(Q, K[perm], V[perm])
    np.testing.assert_allclose(O, O3, rtol=1e-12, atol=1e-12)


def test_dense_dominant_key_selects_its_value():
    L, d = 10, 8
    Q = np.zeros((1, d), np.float32); Q[0, 0] = 100.0
    K = np.zeros((L, d), np.float32); K[7, 0] = 10.0
    V = np.arange(L * d, dtype=np.float32).reshape(L, d)
    O = oracle.dense_rows(np.concatenate([Q, np.zeros((L - 1, d), np.float32)]), K, V, 0, 1)
    np.testing.assert_allclose(O[0], V[7], rtol=0, atol=1e-100 + 1e-120)

"""Pins for the oracle's reweighted block attention (AB-Attention page, SIP item
and "Donanım Dostu Çekirdek" item) and its reduction to dense attention.

* With every block kept at pi = 1 it is dense softmax(QK^T/sqrt(d))V
  (torch SDPA in fp64), ragged last KV block and query block included.
* A weight 1/pi_j = w (an integer) is the same as repeating block j's keys
  and values w times in a dense attention over the kept blocks (SDPA, fp64).
* An empty list gives zeros; the list order does not matter.
"""
import numpy as np
import pytest
import torch

import oracle

TWO32 = 1 << 32


def _sdpa64(q, K, V):
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(K), t(V))[0, 0].numpy()


def _qkv(L, d, seed):
    rng = np.random.default_rng(seed)
    Q = (rng.standard_normal((L, d)) * 1.5).astype(np.float32)
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = rng.standard_normal((L, d)).astype(np.float32)
    return Q, K, V


@pytest.mark.parametrize("L,d,qb,kb", [(64, 16, 64, 16), (100, 32, 64, 16), (77, 64, 128, 32),
                                       (130, 128, 128, 64)])
def test_full_list_with_unit_pi_is_dense(L, d, qb, kb):
    Q, K, V = _qkv(L, d, L + d)
    Nkv = -(-L // kb)
    idx = np.arange(Nkv, dtype=np.int32)
    pq = np.zeros(Nkv, np.uint32)
    ref = _sdpa64(Q, K, V)
    for i in range(-(-L // qb)):
        O = oracle.ht_attention_block(Q, K, V, qb, kb, i, idx, pq, Nkv)
        np.testing.assert_allclose(O, ref[i * qb: min(L, (i + 1) * qb)], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(O, oracle.dense_rows(Q, K, V, i * qb, O.shape[0]), rtol=1e-11,
                                   atol=1e-12)


def test_integer_weights_equal_repeated_blocks():
    L, d, qb, kb = 96, 16, 32, 8
    Q, K, V = _qkv(L, d, 21)
    sel = np.array([0, 3, 4, 9, 11], np.int32)
    w = np.array([1, 2, 4, 8, 1], np.int64)          # 1/pi
    pq = np.array([(TWO32 // int(x)) % TWO32 for x in w], np.uint32)
    Kr = np.concatenate([np.repeat(K[j * kb:(j + 1) * kb][None], x, 0).reshape(-1, d)
                         for j, x in zip(sel, w)])
    Vr = np.concatenate([np.repeat(V[j * kb:(j + 1) * kb][None], x, 0).reshape(-1, d)
                         for j, x in zip(sel, w)])
    for i in range(L // qb):
        O = oracle.ht_attention_block(Q, K, V, qb, kb, i, sel, pq, len(sel))
        np.testing.assert_allclose(O, _sdpa64(Q[i * qb:(i + 1) * qb], Kr, Vr), rtol=1e-11, atol=1e-12)


def test_ragged_last_kv_block_excludes_keys_beyond_L():
    L, d, qb, kb = 70, 16, 64, 16           # last KV block has 6 keys, last query block 6 rows
    Q, K, V = _qkv(L, d, 22)
    sel = np.array([1, 4], np.int32)
    pq = np.zeros(2, np.uint32)
    keys = np.r_[16:32, 64:70]
    for i in range(2):
        O = oracle.ht_attention_block(Q, K, V, qb, kb, i, sel, pq, 2)
        np.testing.assert_allclose(O, _sdpa64(Q[i * qb: min(L, (i + 1) * qb)], K[keys], V[keys]),
                                   rtol=1e-11, atol=1e-12)


def test_empty_list_gives_zero_and_order_does_not_matter():
    L, d = 64, 16
    Q, K, V = _qkv(L, d, 23)
    O = oracle.ht_attention_block(Q, K, V, 64, 16, 0, np.zeros(0, np.int32), np.zeros(0, np.uint32), 0)
    assert O.shape == (64, 16) and not O.any()
    sel = np.array([0, 2, 3], np.int32)
    pq = np.array([123456789, 0, 3000000000], np.uint32)
    a = oracle.ht_attention_block(Q, K, V, 64, 16, 0, sel, pq, 3)
    b = oracle.ht_attention_block(Q, K, V, 64, 16, 0, sel[::-1].copy(), pq[::-1].copy(), 3)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)

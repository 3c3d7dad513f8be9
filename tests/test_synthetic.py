"""The seeded input generators (no method arithmetic): shapes, dtypes,
determinism, and the recipe's stated statistics."""
import numpy as np
import torch

from block_sparse_attention_queries_b200.synthetic import WORKLOADS, make_cross_qkv, make_qkv, make_workload_qkv


def test_shapes_dtypes_and_determinism():
    Q, K, V = make_qkv(1, 2, (2, 8, 8), 64, 8, seed=7)
    assert Q.shape == K.shape == V.shape == (1, 2, 128, 64) and Q.dtype == torch.bfloat16
    Q2, K2, V2 = make_qkv(1, 2, (2, 8, 8), 64, 8, seed=7)
    assert torch.equal(Q, Q2) and torch.equal(K, K2) and torch.equal(V, V2)
    Q3, _, _ = make_qkv(1, 2, (2, 8, 8), 64, 8, seed=8)
    assert not torch.equal(Q, Q3)


def test_cross_generator_shapes_and_determinism():
    Q, K, V = make_cross_qkv(2, 1, (2, 8, 8), (3, 5, 7), 64, 8, seed=3)
    assert Q.shape == (2, 1, 128, 64) and K.shape == V.shape == (2, 1, 105, 64)
    Qb, Kb, Vb = make_cross_qkv(2, 1, (2, 8, 8), (3, 5, 7), 64, 8, seed=3)
    assert torch.equal(Q, Qb) and torch.equal(K, Kb) and torch.equal(V, Vb)
    w = WORKLOADS["cross_long"]
    Qw, Kw, Vw = make_workload_qkv(w)
    assert Qw.shape == (w.B, w.H, w.L, w.d) and Kw.shape == (w.B, w.H, w.Lk, w.d)


def test_recipe_statistics():
    # a token's q.k/sqrt(d) with its own key is about s_peak (8) on average;
    # V is N(0,1) with about 1 % of the tokens scaled by 10
    Q, K, V = make_qkv(1, 4, (4, 16, 16), 128, 16, seed=11)
    q = Q.double()[0]
    k = K.double()[0]
    self_logit = (q * k).sum(-1) / np.sqrt(128)
    assert 6.0 < float(self_logit.mean()) < 10.0
    rms = V.double()[0].pow(2).mean(-1).sqrt()
    frac = float((rms > 5).double().mean())
    assert 0.003 < frac < 0.02

"""Pins for the oracle's SIP (AB-Attention page, "AB-Attention ve Üç Temel
Yeniliği", SIP item): budget, inclusion probabilities with capping, the
Bernoulli draw and the 1/pi-weighted (Horvitz-Thompson) sums.

Pins: an independent exact construction of the capped probabilities
(enumerating the number of capped blocks, in integers), closed forms, exact
enumeration of all 2^12 samples of a 12-block row (unbiasedness to 1e-12),
Monte Carlo over 4096 seeds, and keep-fraction bounds.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_queries_b200.synthetic import WORKLOADS, make_workload_qkv

TWO32 = 1 << 32


def _W(P):
    P = np.asarray(P, np.float32).astype(np.float64)
    return np.maximum(1, np.floor(P * 2.0 ** 24)).astype(np.int64)


def _pps_reference(W, Kb):
    """Capped inclusion probabilities min(1, c W_j) with sum Kb, found by trying
    every number k of capped blocks (the k largest W) and checking that the
    implied c = (Kb - k) / (sum of the rest) caps exactly those.  Returns the
    capped mask and the exact rational c."""
    W = [int(w) for w in W]
    order = sorted(range(len(W)), key=lambda j: -W[j])
    total = sum(W)
    for k in range(0, Kb + 1):
        rest = total - sum(W[order[t]] for t in range(k))
        if rest == 0:
            continue
        c = Fraction(Kb - k, rest)
        ok_capped = all(c * W[order[t]] >= 1 for t in range(k))
        ok_free = all(c * W[order[t]] < 1 for t in range(k, len(W)))
        if ok_capped and ok_free:
            capped = np.zeros(len(W), bool)
            capped[order[:k]] = True
            return capped, c
    raise AssertionError("no capping level found")


def _skewed_rows(n_rows, Nkv, seed):
    rng = np.random.default_rng(seed)
    rows = []
    for r in range(n_rows):
        x = rng.standard_normal(Nkv) * (1 + r % 4) * 1.5
        p = np.exp(x - x.max())
        rows.append((p / p.sum()).astype(np.float32))
    return rows


def test_budget_values():
    assert oracle.budget(64, 0.10) == 6
    assert oracle.budget(512, 0.10) == 51
    assert oracle.budget(512, 1.0) == 512
    assert oracle.budget(2048, 0.11) == 225
    assert oracle.budget(7425, 0.08) == 594     # ceil would give 595 from binary rounding
    assert oracle.budget(4725, 0.05) == 236
    assert oracle.budget(10, 1e-6) == 1
    assert oracle.budget(10, 1.0) == 10


@pytest.mark.parametrize("Nkv,Kb", [(64, 6), (512, 51), (300, 150), (33, 1), (200, 199)])
def test_inclusion_probabilities_exact_against_capping_construction(Nkv, Kb):
    for r, P in enumerate(_skewed_rows(6, Nkv, Nkv + Kb)):
        _, _, _, Pi = oracle.sip_row(P, Kb, 1, 0, 0, r, want_pi=True)
        Pi = Pi.astype(object)
        W = _W(P)
        capped, c = _pps_reference(W, Kb)
        for j in range(Nkv):
            if capped[j]:
                assert Pi[j] == TWO32
            else:
                exact = c * int(W[j]) * TWO32
                assert Pi[j] == max(1, exact.numerator // exact.denominator)
        total = sum(int(x) for x in Pi)
        assert abs(total - Kb * TWO32) <= Nkv
        assert all(1 <= int(x) <= TWO32 for x in Pi)


def test_inclusion_probabilities_monotone_in_weight():
    for P in _skewed_rows(4, 257, 3):
        _, _, _, Pi = oracle.sip_row(P, 40, 7, 0, 0, 0, want_pi=True)
        W = _W(P)
        o = np.argsort(W, kind="stable")
        assert np.all(np.diff(Pi[o].astype(np.float64)) >= 0)


def test_uniform_and_full_budget_closed_forms():
    Nkv = 100
    P = np.full(Nkv, 1.0 / Nkv, np.float32)
    _, _, _, Pi = oracle.sip_row(P, 13, 5, 0, 0, 0, want_pi=True)
    assert np.all(Pi == (13 * TWO32) // Nkv)
    P = _skewed_rows(1, Nkv, 9)[0]
    idx, pq, n, Pi = oracle.sip_row(P, Nkv, 5, 0, 0, 0, want_pi=True)
    assert n == Nkv and np.all(Pi == TWO32) and np.all(pq == 0)
    np.testing.assert_array_equal(idx, np.arange(Nkv))


def test_draw_rule_and_ascending_lists():
    P = _skewed_rows(1, 130, 11)[0]
    seed, b, h, i = 0x0123456789ABCDEF, 2, 3, 17
    idx, pq, n, Pi = oracle.sip_row(P, 20, seed, b, h, i, want_pi=True)
    key = [seed & 0xFFFFFFFF, seed >> 32]
    kept = []
    for j in range(130):
        u = int(oracle.philox4x32_10([j >> 2, i, h, b], key)[j & 3])
        if u < int(Pi[j]):
            kept.append(j)
    np.testing.assert_array_equal(idx, kept)
    np.testing.assert_array_equal(pq, [int(Pi[j]) % TWO32 for j in kept])
    assert np.all(np.diff(idx) > 0)


def _tiny_P():
    w = WORKLOADS["tiny"]
    Q, K, _ = make_workload_qkv(w)
    return oracle.select_head(Q[0, 0].float().numpy(), K[0, 0].float().numpy(), w.q_block,
                              w.kv_block, w.C, w.kmeans_iters).astype(np.float32), w


@pytest.mark.slow
def test_monte_carlo_inclusion_frequency_and_keep_fraction():
    P, w = _tiny_P()
    Nq, Nkv = P.shape
    Kb = oracle.budget(Nkv, w.keep_ratio)
    S = 4096
    freq = np.zeros((Nq, Nkv))
    counts = np.zeros((S, Nq))
    Pi = np.stack([oracle.sip_row(P[i], Kb, 0, 0, 0, i, want_pi=True)[3] for i in range(Nq)])
    pi = Pi.astype(np.float64) / TWO32
    for s in range(S):
        for i in range(Nq):
            idx, _, n = oracle.sip_row(P[i], Kb, s, 0, 0, i)
            freq[i, idx] += 1
            counts[s, i] = n
    freq /= S
    se = np.sqrt(pi * (1 - pi) / S)
    assert np.all(np.abs(freq - pi) <= 5 * se + 1.0 / S)
    # expected count: sum of pi is Kb per row
    np.testing.assert_allclose(pi.sum(1), Kb, atol=Nkv / TWO32)
    # keep fraction: the per-seed total count has mean sum(pi), var sum pi(1-pi)
    tot = counts.sum(1)
    sd = np.sqrt((pi * (1 - pi)).sum())
    assert abs(tot.mean() - pi.sum()) <= 5 * sd / np.sqrt(S)
    assert np.all(np.abs(tot - pi.sum()) <= 6 * sd + 1)


def test_exact_enumeration_horvitz_thompson_is_unbiased():
    # 12 KV blocks of 4 keys: enumerate all 2^12 samples with probability
    # prod(pi) prod(1 - pi); the expected weighted numerator and denominator
    # equal the dense sums (fixed shift), to 1e-12.
    rng = np.random.default_rng(12)
    nb, bs, d = 12, 4, 8
    L = nb * bs
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = rng.standard_normal((L, d)).astype(np.float32)
    q = (rng.standard_normal(d) * 2).astype(np.float32)
    P = _skewed_rows(1, nb, 13)[0]
    _, _, _, Pi = oracle.sip_row(P, 4, 0, 0, 0, 0, want_pi=True)
    pi = Pi.astype(np.float64) / TWO32
    pq = (Pi % TWO32).astype(np.uint32)
    s = K.astype(np.float64) @ q.astype(np.float64) / np.sqrt(d)
    m = s.max()
    dense_den = np.exp(s - m).sum()
    dense_num = (np.exp(s - m)[:, None] * V.astype(np.float64)).sum(0)
    e_num = np.zeros(d)
    e_den = 0.0
    tot_prob = 0.0
    for mask in range(1 << nb):
        sel = [j for j in range(nb) if mask >> j & 1]
        prob = np.prod([pi[j] if mask >> j & 1 else 1 - pi[j] for j in range(nb)])
        if prob == 0.0:
            continue
        tot_prob += prob
        if not sel:
            continue
        num, den = oracle.ht_sums(q, K, V, bs, np.array(sel, np.int32), pq[sel], m)
        e_num += prob * num
        e_den += prob * den
    assert abs(tot_prob - 1) < 1e-12
    np.testing.assert_allclose(e_den, dense_den, rtol=1e-12)
    np.testing.assert_allclose(e_num, dense_num, rtol=1e-11, atol=1e-12 * np.abs(dense_num).max())
    # and the ratio of expectations is the dense attention output (torch SDPA, fp64)
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.astype(np.float64))[None, None, None],
        torch.from_numpy(K.astype(np.float64))[None, None],
        torch.from_numpy(V.astype(np.float64))[None, None])[0, 0, 0].numpy()
    np.testing.assert_allclose(e_num / e_den, o, rtol=1e-11, atol=1e-12)


@pytest.mark.slow
def test_monte_carlo_horvitz_thompson_sums_on_tiny_workload():
    w = WORKLOADS["tiny"]
    Q, K, V = (t[0, 0].float().numpy() for t in make_workload_qkv(w))
    P, _ = _tiny_P()
    Nkv = P.shape[1]
    Kb = oracle.budget(Nkv, w.keep_ratio)
    d = w.d
    for (i, r) in [(0, 5), (7, 33), (15, 63)]:
        q = Q[i * w.q_block + r]
        s = K.astype(np.float64) @ q.astype(np.float64) / np.sqrt(d)
        m = s.max()
        den_ref = np.exp(s - m).sum()
        num_ref = (np.exp(s - m)[:, None] * V.astype(np.float64)).sum(0)
        S = 4096
        nums = np.zeros((S, d))
        dens = np.zeros(S)
        for seed in range(S):
            idx, pq, n = oracle.sip_row(P[i], Kb, seed, 0, 0, i)
            if n:
                nums[seed], dens[seed] = oracle.ht_sums(q, K, V, w.kv_block, idx, pq, m)
        se_den = dens.std(ddof=1) / np.sqrt(S)
        assert abs(dens.mean() - den_ref) <= 5 * se_den
        se_num = nums.std(0, ddof=1) / np.sqrt(S)
        assert np.all(np.abs(nums.mean(0) - num_ref) <= 5 * se_num + 1e-12)

"""Pins of the oracle's systematic sampling (a fixed-size alternative to
SIP's independent draws, with the same inclusion probabilities).

AB-Attention page, section "AB-Attention ve Üç Temel Yeniliği", SIP item:
blocks are sampled in proportion to the IBCS estimate and reweighted by the
inverse inclusion probability; the sampling design itself is left open.
The selection as a function of the offset U in [0, 2^32) is piecewise
constant, changing only where U crosses C_j mod 2^32 (C_j = cumulative Pi);
enumerating those pieces gives exact expectations:
* every block is kept with probability exactly Pi_j / 2^32;
* the 1/pi-weighted numerator and denominator are unbiased (exactly), and
  their ratio of expectations is dense attention (torch SDPA);
* the sample size is floor or ceil of sum Pi / 2^32; uniform Pi gives the
  textbook every-k-th selection; capped blocks are always kept;
* the seeded form takes U from word 0 of Philox4x32-10 at counter
  (0xFFFFFFFF, i, h, b) (Philox is pinned against cuRAND elsewhere)."""
import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")
TWO32 = float(2 ** 32)


def _rows(n, Nkv, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, Nkv)) * rng.uniform(0.5, 4.0, (n, 1))
    P = np.exp(x - x.max(-1, keepdims=True))
    return (P / P.sum(-1, keepdims=True)).astype(np.float32)


def _pieces(Pi):
    """Breakpoints of the selection in U: the distinct C_j mod 2^32, with 0 and 2^32."""
    C = np.concatenate([[0], np.cumsum(Pi.astype(object))])
    cuts = sorted({int(c) % 2 ** 32 for c in C} | {0, 2 ** 32})
    return [(lo, hi) for lo, hi in zip(cuts[:-1], cuts[1:]) if hi > lo]


@pytest.mark.parametrize("Nkv,Kb,seed", [(12, 4, 1), (40, 7, 2), (64, 6, 3), (31, 30, 4)])
def test_inclusion_probabilities_exact_by_enumerating_offsets(Nkv, Kb, seed):
    P = _rows(1, Nkv, seed)[0]
    _, _, _, Pi = oracle.sip_row(P, Kb, 0, 0, 0, 0, want_pi=True)
    freq = np.zeros(Nkv)
    sizes = set()
    for lo, hi in _pieces(Pi):
        idx, pq, n = oracle.systematic_row_u(P, Kb, lo)
        assert oracle.systematic_row_u(P, Kb, hi - 1)[2] == n  # constant on the piece
        np.testing.assert_array_equal(oracle.systematic_row_u(P, Kb, hi - 1)[0], idx)
        freq[idx] += (hi - lo) / TWO32
        sizes.add(n)
        np.testing.assert_array_equal(pq, (Pi[idx] % 2 ** 32).astype(np.uint32))
        assert np.all(np.diff(idx) > 0)
    np.testing.assert_allclose(freq, Pi.astype(np.float64) / TWO32, rtol=0, atol=1e-15)
    total = float(Pi.astype(np.float64).sum()) / TWO32
    assert sizes <= {int(np.floor(total)), int(np.ceil(total))}


def test_horvitz_thompson_exact_under_systematic_sampling():
    rng = np.random.default_rng(12)
    nb, bs, d = 12, 4, 8
    L = nb * bs
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = rng.standard_normal((L, d)).astype(np.float32)
    q = (rng.standard_normal(d) * 2).astype(np.float32)
    P = _rows(1, nb, 13)[0]
    Kb = 4
    _, _, _, Pi = oracle.sip_row(P, Kb, 0, 0, 0, 0, want_pi=True)
    s = K.astype(np.float64) @ q.astype(np.float64) / np.sqrt(d)
    m = s.max()
    dense_den = np.exp(s - m).sum()
    dense_num = (np.exp(s - m)[:, None] * V.astype(np.float64)).sum(0)
    e_num, e_den, tot = np.zeros(d), 0.0, 0.0
    for lo, hi in _pieces(Pi):
        w = (hi - lo) / TWO32
        idx, pq, n = oracle.systematic_row_u(P, Kb, lo)
        tot += w
        num, den = oracle.ht_sums(q, K, V, bs, idx, pq, m)
        e_num += w * num
        e_den += w * den
    assert abs(tot - 1) < 1e-15
    np.testing.assert_allclose(e_den, dense_den, rtol=1e-12)
    np.testing.assert_allclose(e_num, dense_num, rtol=1e-11, atol=1e-12 * np.abs(dense_num).max())
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.astype(np.float64))[None, None, None],
        torch.from_numpy(K.astype(np.float64))[None, None],
        torch.from_numpy(V.astype(np.float64))[None, None])[0, 0, 0].numpy()
    np.testing.assert_allclose(e_num / e_den, o, rtol=1e-11, atol=1e-12)


def test_uniform_probabilities_give_every_kth_block():
    Nkv, Kb = 64, 8
    P = np.full(Nkv, 1.0 / Nkv, np.float32)
    for U in (0, 12345, 2 ** 31, 2 ** 32 - 1):
        idx, _, n = oracle.systematic_row_u(P, Kb, U)
        assert n == Kb
        np.testing.assert_array_equal(np.diff(idx), np.full(Kb - 1, Nkv // Kb))  # textbook systematic sample
        assert idx[0] == U >> 29  # Pi_j = 2^29: the first point U lies in block floor(U / 2^29)


def test_capped_blocks_always_kept_and_sizes():
    P = _rows(8, 512, 5)
    Kb = 51
    for r in range(8):
        _, _, _, Pi = oracle.sip_row(P[r], Kb, 0, 0, 0, 0, want_pi=True)
        capped = np.nonzero(Pi == 2 ** 32)[0]
        for seed in range(5):
            idx, _, n = oracle.systematic_row(P[r], Kb, seed, 0, 1, r)
            assert set(capped.tolist()) <= set(idx.tolist())
            assert Kb - 1 <= n <= Kb


def test_seeded_offset_is_philox_word0_at_counter_ffffffff():
    P = _rows(1, 300, 9)[0]
    for (seed, b, h, i) in [(42, 0, 0, 0), (2 ** 63 + 5, 1, 3, 17), (7, 0, 39, 255)]:
        key = np.array([seed & 0xFFFFFFFF, seed >> 32], np.uint32)
        U = int(oracle.philox4x32_10(np.array([0xFFFFFFFF, i, h, b], np.uint32), key)[0])
        a = oracle.systematic_row(P, 30, seed, b, h, i)
        e = oracle.systematic_row_u(P, 30, U)
        np.testing.assert_array_equal(a[0], e[0])
        assert a[2] == e[2]

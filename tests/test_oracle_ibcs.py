"""Pins for the oracle's IBCS (AB-Attention page, "AB-Attention ve Üç Temel
Yeniliği", IBCS item): KV-block summaries, per-query-block k-means and the
block-mass estimate.

Pinned by invariants of Lloyd's algorithm, scikit-learn's Lloyd k-means from
the same initial centroids (a library routine), special cases that reduce to
a textbook softmax (scipy), and closed forms.
"""
import numpy as np
import pytest
from scipy.special import softmax
from sklearn.cluster import KMeans

import oracle


def _strided_init_rows(n, C):
    return [int(np.floor((c + 0.5) * n / C)) for c in range(C)]


# ----------------------------------------------------------------- summaries

@pytest.mark.parametrize("L,bs", [(64, 16), (70, 16), (33, 32), (5, 16)])
def test_ksum_is_mean_of_valid_keys(L, bs):
    rng = np.random.default_rng(L)
    K = rng.standard_normal((L, 8)).astype(np.float32)
    S = oracle.ksum(K, bs)
    assert S.shape == (-(-L // bs), 8)
    for j in range(S.shape[0]):
        blk = K[j * bs: min(L, (j + 1) * bs)].astype(np.float64)
        np.testing.assert_allclose(S[j], blk.mean(0), rtol=1e-14, atol=1e-15)


# ------------------------------------------------------------------- k-means

def _objective(X, mu, assign):
    return float(((X.astype(np.float64) - mu[assign]) ** 2).sum())


@pytest.mark.parametrize("n,C", [(128, 8), (120, 8), (64, 4), (80, 16), (16, 8)])
def test_kmeans_lloyd_invariants(n, C):
    rng = np.random.default_rng(n * 31 + C)
    X = (rng.standard_normal((n, 16)) + rng.integers(0, 3, (n, 1))).astype(np.float32)
    prev_obj = np.inf
    for T in range(1, 6):
        mu, cnt, a = oracle.kmeans(X, C, T, return_assign=True)
        # counts are the sizes of the last assignment
        np.testing.assert_array_equal(cnt, np.bincount(a, minlength=C))
        # every non-empty centroid is the mean of its members
        for c in range(C):
            if cnt[c]:
                np.testing.assert_allclose(mu[c], X[a == c].astype(np.float64).mean(0), rtol=1e-12,
                                           atol=1e-12)
        # the last assignment is an argmin against the previous centroids
        mu_prev = (np.asarray(X[_strided_init_rows(n, C)], np.float64) if T == 1
                   else oracle.kmeans(X, C, T - 1)[0])
        dist = ((X[:, None, :].astype(np.float64) - mu_prev[None]) ** 2).sum(-1)
        best = dist.min(1)
        assert np.all(dist[np.arange(n), a] <= best + 1e-9)
        # Lloyd's objective never increases
        obj = _objective(X, mu, a)
        assert obj <= prev_obj + 1e-9
        prev_obj = obj


def test_kmeans_c1_is_block_mean():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((100, 32)).astype(np.float32)
    mu, cnt = oracle.kmeans(X, 1, 3)
    np.testing.assert_allclose(mu[0], X.astype(np.float64).mean(0), rtol=1e-13, atol=1e-14)
    assert cnt[0] == 100


def test_kmeans_c_equals_n_returns_the_queries():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((8, 16)).astype(np.float32)
    mu, cnt = oracle.kmeans(X, 8, 3)
    np.testing.assert_array_equal(mu, X.astype(np.float64))
    np.testing.assert_array_equal(cnt, np.ones(8))


def test_kmeans_recovers_separated_clumps():
    # C contiguous clumps of n/C queries far apart: the strided init takes one
    # query from each clump, so one iteration already gives the clump means.
    rng = np.random.default_rng(4)
    C, m, d = 8, 16, 32
    centers = rng.standard_normal((C, d)) * 50
    X = np.concatenate([centers[c] + rng.standard_normal((m, d)) for c in range(C)]).astype(np.float32)
    mu, cnt = oracle.kmeans(X, C, 3)
    for c in range(C):
        np.testing.assert_allclose(mu[c], X[c * m:(c + 1) * m].astype(np.float64).mean(0), rtol=1e-12)
    np.testing.assert_array_equal(cnt, np.full(C, m))


def test_kmeans_tie_goes_to_lowest_cluster():
    # two identical initial centroids: every query ties, all go to cluster 0,
    # cluster 1 stays empty and keeps its centroid.
    X = np.array([[1.0, 0.0]] * 3 + [[1.0, 0.0]] + [[3.0, 0.0]] * 4, np.float32)
    # init rows for n=8, C=2 are 2 and 6 -> (1,0) and (3,0): make them equal
    X[6] = X[2]
    mu, cnt, a = oracle.kmeans(X, 2, 1, return_assign=True)
    assert (a == 0).all() and cnt[1] == 0
    np.testing.assert_array_equal(mu[1], X[2].astype(np.float64))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_kmeans_matches_sklearn_lloyd(seed):
    rng = np.random.default_rng(100 + seed)
    n, d, C, T = 128, 16, 8, 3
    X = (rng.standard_normal((n, d)) + 4 * rng.integers(0, 4, (n, d))).astype(np.float32)
    init = X[_strided_init_rows(n, C)].astype(np.float64)
    km = KMeans(n_clusters=C, init=init, n_init=1, max_iter=T, tol=0.0, algorithm="lloyd")
    km.fit(X.astype(np.float64))
    mu, _ = oracle.kmeans(X, C, T)
    # sklearn stops early only at a fixed point, where more Lloyd steps change nothing
    np.testing.assert_allclose(mu, km.cluster_centers_, rtol=1e-9, atol=1e-9)


# ---------------------------------------------------------------- block mass

def test_block_mass_c1_bk1_is_softmax_of_mean_query():
    # one cluster and one key per KV block: P = softmax_j(qbar . k_j / sqrt(d))
    rng = np.random.default_rng(7)
    L, d = 50, 16
    Q = rng.standard_normal((L, d)).astype(np.float32)
    K = rng.standard_normal((L, d)).astype(np.float32)
    P = oracle.select_head(Q, K, q_block=L, kv_block=1, C=1, iters=3)
    qbar = Q.astype(np.float64).mean(0)
    np.testing.assert_allclose(P[0], softmax(K.astype(np.float64) @ qbar / np.sqrt(d)), rtol=1e-12)


def test_block_mass_equal_keys_is_block_share():
    # identical keys: every score is the same up to ln n_j, so P_j = n_j / L
    L, d, bs = 100, 8, 16
    rng = np.random.default_rng(8)
    Q = rng.standard_normal((L, d)).astype(np.float32)
    K = np.tile(rng.standard_normal((1, d)).astype(np.float32), (L, 1))
    P = oracle.select_head(Q, K, q_block=32, kv_block=bs, C=4, iters=3)
    n_j = np.array([min(bs, L - j * bs) for j in range(-(-L // bs))], np.float64)
    for row in P:
        np.testing.assert_allclose(row, n_j / L, rtol=1e-12)


def test_block_mass_two_clumps_mixes_by_cluster_share():
    # two well separated query clumps of sizes 24 and 8: the centroids are the
    # clump means and P = (24/32) softmax(mu1 . kbar) + (8/32) softmax(mu2 . kbar)
    rng = np.random.default_rng(9)
    d, bs, L = 16, 4, 32
    c1, c2 = rng.standard_normal(d) * 40, rng.standard_normal(d) * 40
    # order so that the strided init (rows 8 and 24 for n=32, C=2) hits each clump
    Q = np.concatenate([c1 + rng.standard_normal((16, d)), c2 + rng.standard_normal((8, d)),
                        c1 + rng.standard_normal((8, d))]).astype(np.float32)
    K = (rng.standard_normal((L, d)) * 0.2).astype(np.float32)
    P = oracle.select_head(Q, K, q_block=L, kv_block=bs, C=2, iters=3)[0]
    m1 = np.concatenate([Q[:16], Q[24:]]).astype(np.float64).mean(0)
    m2 = Q[16:24].astype(np.float64).mean(0)
    kbar = K.astype(np.float64).reshape(L // bs, bs, d).mean(1)
    ref = 0.75 * softmax(kbar @ m1 / 4.0) + 0.25 * softmax(kbar @ m2 / 4.0)
    np.testing.assert_allclose(P, ref, rtol=1e-11)


def test_block_mass_rows_sum_to_one_and_key_shift_invariance():
    rng = np.random.default_rng(10)
    L, d = 300, 32
    Q = rng.standard_normal((L, d)).astype(np.float32)
    K = (np.round(rng.standard_normal((L, d)) * 64) / 64).astype(np.float32)
    P = oracle.select_head(Q, K, q_block=64, kv_block=16, C=4, iters=3)
    np.testing.assert_allclose(P.sum(1), 1.0, atol=1e-12)
    P2 = oracle.select_head(Q, K + np.float32(0.5), q_block=64, kv_block=16, C=4, iters=3)
    np.testing.assert_allclose(P, P2, rtol=1e-9, atol=1e-15)


def test_select_head_row_subset_and_centroid_outputs():
    rng = np.random.default_rng(11)
    L, d = 200, 16
    Q = rng.standard_normal((L, d)).astype(np.float32)
    K = rng.standard_normal((L, d)).astype(np.float32)
    P, mu, cnt = oracle.select_head(Q, K, 64, 16, 4, 3, want_centroids=True)
    Ps, mus, cnts = oracle.select_head(Q, K, 64, 16, 4, 3, rows=[3, 1], want_centroids=True)
    np.testing.assert_array_equal(Ps, P[[3, 1]])
    np.testing.assert_array_equal(mus, mu[[3, 1]])
    assert cnt[3].sum() == 200 - 3 * 64 and cnt[1].sum() == 64

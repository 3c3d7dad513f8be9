"""Shared helpers of the GPU parity tests: conversions, error metrics and
oracle runs over many independent (b, h, query block) units."""
from __future__ import annotations

import numpy as np

import oracle

MAX_ABS = 2e-2   # attention output vs the fp64 oracle, on top of bf16 output rounding
REL_L2 = 5e-3
BF16_HALF_ULP_REL = 2.0 ** -8  # round-to-nearest bf16 (8 significant bits): |x - bf16(x)| <= 2^-8 |x|


def np32(t):
    return t.detach().float().cpu().numpy()


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_close_attention(got, ref, what=""):
    """Element-wise |got - ref| <= 2e-2 + 2^-8 |ref| and rel-L2 <= 5e-3.

    The bf16 output format alone rounds a value x by up to 2^-8 |x| (0.031 at
    |x| = 8), so the 2e-2 absolute bound is applied on top of that rounding."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if not got.size:
        return 0.0, 0.0
    diff = np.abs(got - ref)
    excess = float((diff - (MAX_ABS + BF16_HALF_ULP_REL * np.abs(ref))).max())
    r = rel_l2(got, ref)
    err = float(diff.max())
    assert excess <= 0 and r <= REL_L2, (
        f"{what}: max-abs {err:.3g} (excess over bound {excess:.3g}) rel-L2 {r:.3g} "
        f"(max|ref| {np.abs(ref).max():.3g})")
    return err, r


def oracle_ht_units(Qn, Kn, Vn, q_block, kv_block, units, idx, pq, cnt, threads=None):
    """Oracle reweighted attention for units [(b, h, i)] on given lists.

    Qn/Kn/Vn: fp32 numpy [B, H, L, d]; idx/pq/cnt numpy list arrays.
    Returns {(b, h, i): O [n_i, d] fp64}."""
    def one(u):
        b, h, i = u
        c = int(cnt[b, h, i])
        return u, oracle.ht_attention_block(Qn[b, h], Kn[b, h], Vn[b, h], q_block, kv_block, i,
                                            idx[b, h, i], pq[b, h, i].astype(np.uint32), c)
    return dict(oracle.run_units(one, list(units), threads))


def oracle_dense_units(Qn, Kn, Vn, q_block, units, threads=None):
    def one(u):
        b, h, i = u
        L = Qn.shape[2]
        n = min(q_block, L - i * q_block)
        return u, oracle.dense_rows(Qn[b, h], Kn[b, h], Vn[b, h], i * q_block, n)
    return dict(oracle.run_units(one, list(units), threads))


def oracle_sip_rows(P, Kb, seed, rows, threads=None):
    """Oracle SIP on fp32 rows P[b, h, i] for rows [(b, h, i)]."""
    def one(u):
        b, h, i = u
        return u, oracle.sip_row(P[b, h, i], Kb, seed, b, h, i)
    return dict(oracle.run_units(one, list(rows), threads))


def selection_agreement(pairs, what=""):
    """Selection of the CUDA path vs the oracle's, aggregated over rows:
    pairs = [(gpu kept blocks, oracle kept blocks), ...].  Asserts and returns
    (agreement, jaccard): agreement = sum |S_gpu & S_oracle| / sum |S_oracle|
    >= 0.995 (the parity contract) and the Jaccard index sum |S_gpu & S_oracle|
    / sum |S_gpu | S_oracle| >= 0.99 (both draws use the same uniforms, so the
    two sets differ only at blocks whose inclusion probability the two
    estimates put on different sides of the draw)."""
    inter = tot = union = 0
    for g, o in pairs:
        a, b = set(np.asarray(g).tolist()), set(np.asarray(o).tolist())
        inter += len(a & b)
        tot += len(b)
        union += len(a | b)
    agree, jac = inter / max(tot, 1), inter / max(union, 1)
    print(f"selection {what}: agreement {agree:.5f}, Jaccard {jac:.5f} over {len(pairs)} rows")
    assert agree >= 0.995, (what, agree)
    assert jac >= 0.99, (what, jac)
    return agree, jac

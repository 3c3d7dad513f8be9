"""How much attention mass IBCS's estimate finds, against the best possible
selection, on the synthetic inputs (information only; CPU, fp64 oracle).

For the tiny workload's shape (1024 tokens, d = 64, query block 64, KV
block 16, C = 4, 10 % of the KV blocks) and the input generator's peak logit
s_peak in {8, 16, 32}, per head:

* the dense attention A = softmax(QK^T / sqrt(d)) and output D = A V;
* truncation by the oracle's IBCS estimate P (the top-Kb blocks of each query
  block) and by the true block mass (the top-Kb blocks of the query block's
  mean attention row): the true mass each keeps and the relative L2 error of
  the attention restricted to it;
* SIP (the oracle's draws on P, three seeds): the relative L2 error of the
  reweighted estimate;
* the effective number of keys per query, 1 / sum_k A_qk^2.

Run:  python -m oracle.quality_sweep
"""
from __future__ import annotations

import numpy as np

import oracle
from block_sparse_attention_queries_b200.synthetic import make_qkv


def sweep(grid=(4, 16, 16), d=64, F=8, q_block=64, kv_block=16, C=4, keep=0.10, heads=2,
          s_peaks=(8.0, 16.0, 32.0), sip_seeds=(1, 2, 3)):
    rows = []
    L = grid[0] * grid[1] * grid[2]
    Nq, Nkv = -(-L // q_block), -(-L // kv_block)
    Kb = oracle.budget(Nkv, keep)
    for s_peak in s_peaks:
        Q, K, V = make_qkv(1, heads, grid, d, F, seed=1234, s_peak=s_peak)
        acc = {"mass_P": [], "mass_true": [], "err_trunc_P": [], "err_trunc_true": [], "err_sip": [],
               "eff_keys": []}
        for h in range(heads):
            Qn, Kn, Vn = (t[0, h].float().numpy() for t in (Q, K, V))
            D = oracle.dense_rows(Qn, Kn, Vn)
            S = Qn.astype(np.float64) @ Kn.astype(np.float64).T / np.sqrt(d)
            A = np.exp(S - S.max(1, keepdims=True))
            A /= A.sum(1, keepdims=True)
            acc["eff_keys"].append(float(np.mean(1.0 / (A ** 2).sum(1))))
            P = oracle.select_head(Qn, Kn, q_block, kv_block, C, 3)
            for name in ("P", "true"):
                O = np.zeros_like(D)
                kept = []
                for i in range(Nq):
                    r0, r1 = i * q_block, min(L, (i + 1) * q_block)
                    mass = np.add.reduceat(A[r0:r1].mean(0), np.arange(0, L, kv_block))
                    if name == "P":
                        idx, pq, n = oracle.topk_row(P[i].astype(np.float32), Kb)
                    else:
                        idx, pq, n = oracle.topk_row(mass.astype(np.float32), Kb)
                    kept.append(float(mass[idx[:n]].sum()))
                    O[r0:r1] = oracle.ht_attention_block(Qn, Kn, Vn, q_block, kv_block, i, idx, pq, n)
                acc["mass_" + name].append(float(np.mean(kept)))
                acc["err_trunc_" + name].append(float(np.linalg.norm(O - D) / np.linalg.norm(D)))
            for sd in sip_seeds:
                O = np.zeros_like(D)
                for i in range(Nq):
                    idx, pq, n = oracle.sip_row(P[i].astype(np.float32), Kb, sd, 0, h, i)
                    O[i * q_block: min(L, (i + 1) * q_block)] = oracle.ht_attention_block(
                        Qn, Kn, Vn, q_block, kv_block, i, idx, pq, n)
                acc["err_sip"].append(float(np.linalg.norm(O - D) / np.linalg.norm(D)))
        rows.append({"s_peak": s_peak, **{k: round(float(np.mean(v)), 3) for k, v in acc.items()}})
    return rows


if __name__ == "__main__":
    for r in sweep():
        print(r, flush=True)

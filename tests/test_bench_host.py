"""Host-side arithmetic of bench.py on CPU: the executed attention flop of a
set of lists (against a direct count over every kept block), the dense
flop of self- and cross-attention, and the config record."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from block_sparse_attention_queries_b200.synthetic import WORKLOADS  # noqa: E402


def _direct(w, cnt, idx):
    tot = 0
    for b in range(w.B):
        for h in range(w.H):
            for i in range(w.Nq):
                n_i = min(w.q_block, w.L - i * w.q_block)
                for j in idx[b, h, i, :cnt[b, h, i]]:
                    tot += 4 * w.d * n_i * min(w.kv_block, w.Lk - int(j) * w.kv_block)
    return float(tot)


def test_executed_flop_matches_direct_count():
    rng = np.random.default_rng(3)
    for name in ("cross_short", "cross_long", "tiny"):
        w = WORKLOADS[name]
        cnt = rng.integers(0, w.Nkv + 1, size=(w.B, w.H, w.Nq)).astype(np.int32)
        cnt[0, 0, 0] = w.Nkv          # a row holding the partial last block
        cnt[-1, -1, -1] = 0           # an empty row
        idx = np.zeros((w.B, w.H, w.Nq, w.Nkv), np.int32)
        for r in np.ndindex(*cnt.shape):
            idx[r][:cnt[r]] = np.sort(rng.choice(w.Nkv, cnt[r], replace=False))
        assert bench.executed_flop(w, cnt, idx) == _direct(w, cnt, idx), name


def test_dense_flop_and_config_of_cross_attention():
    w = WORKLOADS["cross_wan480"]
    assert (w.L, w.Lk) == (32760, 14040)
    assert bench.dense_flop(w) == 4.0 * 40 * 32760 * 14040 * 128
    s = WORKLOADS["wan480"]
    assert bench.dense_flop(s) == 4.0 * 40 * 32760 ** 2 * 128
    c = bench.config_dict(w)
    assert c["L_kv"] == 14040 and c["grid_kv_txy"] == [9, 30, 52]
    assert "L_kv" not in bench.config_dict(s)
    assert c["l2"].startswith("inputs larger than L2")


def test_tile_flop_counts_full_tiles():
    w = WORKLOADS["cross_short"]                      # kv_block 16: 8 blocks per 128-key tile
    cnt = np.array([[[0, 1, 8, 9, 16, 17]]], np.int32)
    tiles = 0 + 1 + 1 + 2 + 2 + 3
    assert bench.tile_flop(w, cnt) == 4.0 * 128 * 128 * w.d * tiles
    w64 = WORKLOADS["cross_short"].with_(kv_block=64)  # 2 blocks per tile
    assert bench.tile_flop(w64, np.array([3, 4, 5])) == 4.0 * 128 * 128 * w64.d * (2 + 2 + 3)
    # never below the algorithmic count of the same lists
    rng = np.random.default_rng(5)
    c = rng.integers(0, w.Nkv + 1, size=(w.B, w.H, w.Nq)).astype(np.int32)
    idx = np.zeros((w.B, w.H, w.Nq, w.Nkv), np.int32)
    for r in np.ndindex(*c.shape):
        idx[r][:c[r]] = np.sort(rng.choice(w.Nkv, c[r], replace=False))
    assert bench.tile_flop(w, c) >= bench.executed_flop(w, c, idx)


def test_ingress_bytes_and_roofline():
    # per CTA two Q tiles; per 128-key tile of a list one K and one V tile of
    # 128 x d bf16 (padding of the last tile included)
    w = WORKLOADS["wan480"].with_(H=1)
    tile = 128 * w.d * 2
    cnt = np.zeros((1, 1, w.Nq), np.int64)
    cnt[0, 0, :3] = [1, 8, 9]  # 1, 1 and 2 tiles of 8 blocks
    assert bench.ingress_bytes(w, cnt) == (1 + 1 + 2) * 2 * tile + w.Nq * tile
    w32 = w.with_(kv_block=32)  # 4 blocks per tile
    assert bench.ingress_bytes(w32, cnt) == (1 + 2 + 3) * 2 * tile + w.Nq * tile
    r = bench.ingress_roofline(w, cnt, 1.0, {"sm_mhz": 1000.0})
    expect = bench.ingress_bytes(w, cnt) / (1e-3 * 1e9 * bench.NUM_SMS)
    assert abs(r["achieved"] - round(expect, 2)) < 1e-9
    assert r["frac"] == round(expect / bench.TMA_INGRESS_B_PER_CLK_SM, 4)
    assert bench.ingress_roofline(w, cnt, 1.0, {"error": "no samples"})["achieved"] is None

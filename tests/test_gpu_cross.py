"""GPU parity for cross-attention: queries from one sequence (L tokens), keys
and values from another (Lk tokens), Cross-Attention glossary page,
"Cross-Attention Nasıl Çalışır?".  Query blocks follow L, KV blocks Lk.

Workloads (seeded, synthetic; see ``synthetic.make_cross_qkv``):
* cross_short: a 8x32x32 clip (8192 queries, d = 128, q_block 128, kv_block
  16, C = 8) attending to a 3x30x37 clip (3330 keys: not a multiple of 8, so
  the K/V copies take the plain 3-D tensor maps; last KV block of 2 keys);
* cross_long: a 3x20x30 clip (1800 queries, d = 64, q_block 64: an odd
  number of query blocks, the last of 8 rows) attending to a 9x24x40 clip
  (8640 keys, kv_block 32, C = 4, B = 2).

Checks, all through the C ABI: P against the oracle's (independent
centroids), the selection against the oracle's own SIP on its P (>= 99.5 %
agreement), the sampler bit for bit on the GPU's P, the sparse attention on
the GPU's lists and the dense kernel against the oracle within the attention
tolerance, full budget equal to dense bit for bit, and the host-buffer entry
point equal to the device path.
"""
import numpy as np
import pytest

import oracle
from helpers import (assert_close_attention, np32, oracle_dense_units, oracle_ht_units, oracle_sip_rows, rel_l2, selection_agreement)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_sparse_attention_queries_b200 as ab  # noqa: E402
from block_sparse_attention_queries_b200.synthetic import WORKLOADS, make_cross_qkv, make_workload_qkv  # noqa: E402


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from block_sparse_attention_queries_b200 import build as abbuild
    abbuild.build()
    ab.lib()
    return torch.device("cuda:0")


def _no_device_error(dev):
    code = ab.device_error(dev)
    assert code == 0, ab.status_string(code)


def _stack(p, res, units):
    out = np.zeros((p.B, p.H, p.L, p.d))
    for (b, h, i) in units:
        o = res[(b, h, i)]
        out[b, h, i * p.q_block: i * p.q_block + o.shape[0]] = o
    return out


@pytest.mark.parametrize("wname", ["cross_short", "cross_long"])
def test_cross_attention_end_to_end(dev, wname):
    w = WORKLOADS[wname]
    p = ab.Params.of(w)
    assert p.L_kv == w.Lk != w.L
    Qc, Kc, Vc = make_workload_qkv(w)
    assert tuple(Kc.shape) == (p.B, p.H, p.Lk, p.d)
    Q, K, V = (t.to(dev) for t in (Qc, Kc, Vc))
    bufs = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    _no_device_error(dev)
    assert tuple(bufs.P.shape) == (p.B, p.H, p.Nq, p.Nkv)
    Qn, Kn, Vn = np32(Qc), np32(Kc), np32(Vc)
    Kb = oracle.budget(p.Nkv, p.keep_ratio)
    assert Kb == ab.budget(p)
    Pg = bufs.P.cpu().numpy()
    gi = bufs.idx.cpu().numpy()
    gp = bufs.pi_q32.cpu().numpy().view(np.uint32)
    gc = bufs.count.cpu().numpy()
    units = [(b, h, i) for b in range(p.B) for h in range(p.H) for i in range(p.Nq)]

    # P from the oracle's own centroids
    Po = np.zeros_like(Pg, dtype=np.float64)
    for b in range(p.B):
        for h in range(p.H):
            Po[b, h] = oracle.select_head(Qn[b, h], Kn[b, h], p.q_block, p.kv_block, p.C, p.kmeans_iters)
            assert rel_l2(Pg[b, h], Po[b, h]) < 2e-2, (wname, b, h, rel_l2(Pg[b, h], Po[b, h]))

    # the sampler on the GPU's P, bit for bit; agreement with the oracle's selection
    sg = oracle_sip_rows(Pg, Kb, p.seed, units)
    so = oracle_sip_rows(Po.astype(np.float32), Kb, p.seed, units)
    for r in units:
        c = int(gc[r])
        assert c == sg[r][2], (wname, r)
        np.testing.assert_array_equal(gi[r][:c], sg[r][0])
        np.testing.assert_array_equal(gp[r][:c], sg[r][1])
    selection_agreement([(gi[r][:int(gc[r])], so[r][0]) for r in units], wname)

    # sparse attention on the GPU's lists
    ref = _stack(p, oracle_ht_units(Qn, Kn, Vn, p.q_block, p.kv_block, units, gi, gp, gc), units)
    assert_close_attention(np32(bufs.O), ref, f"{wname} sparse")

    # dense cross-attention on the first, a middle and the last query block of every head
    Od = ab.ab_attention_dense(p, Q, K, V)
    torch.cuda.synchronize()
    _no_device_error(dev)
    some = [(b, h, i) for b in range(p.B) for h in range(p.H) for i in sorted({0, p.Nq // 2, p.Nq - 1})]
    refd = oracle_dense_units(Qn, Kn, Vn, p.q_block, some)
    for (b, h, i) in some:
        o = refd[(b, h, i)]
        got = np32(Od[b, h, i * p.q_block: i * p.q_block + o.shape[0]])
        assert_close_attention(got, o, f"{wname} dense b={b} h={h} i={i}")


@pytest.mark.parametrize("wname", ["cross_short", "cross_long"])
def test_cross_full_budget_equals_dense_bitwise(dev, wname):
    w = WORKLOADS[wname]
    p = ab.Params.of(w, keep_ratio=1.0)
    Q, K, V = (t.to(dev) for t in make_workload_qkv(w))
    bufs = ab.ab_forward(p, Q, K, V)
    Od = ab.ab_attention_dense(p, Q, K, V)
    torch.cuda.synchronize()
    _no_device_error(dev)
    assert (bufs.count == p.Nkv).all()
    assert (bufs.pi_q32 == 0).all()
    assert torch.equal(bufs.O, Od)


@pytest.mark.parametrize("B,H,grid,grid_kv", [(1, 9, (2, 12, 20), (3, 10, 11)), (2, 3, (2, 16, 16), (1, 8, 8))])
def test_cross_forward_host_equals_device_path(dev, B, H, grid, grid_kv):
    # 9 heads: pipelined head groups (K/V offsets follow Lk, Q/O offsets L);
    # 6 heads with B = 2: one group of 4 and one of 2
    L = grid[0] * grid[1] * grid[2]
    Lk = grid_kv[0] * grid_kv[1] * grid_kv[2]
    p = ab.Params(B=B, H=H, L=L, d=128, q_block=128, kv_block=16, C=8, keep_ratio=0.2, seed=77, L_kv=Lk)
    Qc, Kc, Vc = make_cross_qkv(B, H, grid, grid_kv, 128, 8, seed=31)
    Q, K, V = (t.to(dev) for t in (Qc, Kc, Vc))
    ref = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    Qh, Kh, Vh = (t.pin_memory() for t in (Qc, Kc, Vc))
    Oh = torch.empty_like(Qc).pin_memory()
    Qd, Kd, Vd = (torch.empty_like(t) for t in (Q, K, V))
    bufs = ab.Buffers(p, dev)
    ab.ab_forward_host(p, Qh, Kh, Vh, Oh, Qd, Kd, Vd, bufs, dev)
    torch.cuda.synchronize()
    _no_device_error(dev)
    assert torch.equal(bufs.count, ref.count)
    assert torch.equal(bufs.idx, ref.idx)
    assert torch.equal(bufs.pi_q32, ref.pi_q32)
    assert torch.equal(bufs.O, ref.O)
    assert torch.equal(Oh, ref.O.cpu())


def test_cross_key_tensor_shape_is_checked(dev):
    w = WORKLOADS["cross_long"]
    p = ab.Params.of(w)
    Q = torch.zeros(p.B, p.H, p.L, p.d, dtype=torch.bfloat16, device=dev)
    K_wrong = torch.zeros(p.B, p.H, p.L, p.d, dtype=torch.bfloat16, device=dev)
    with pytest.raises(ValueError):
        ab.ab_attention_dense(p, Q, K_wrong, K_wrong)

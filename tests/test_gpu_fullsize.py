"""GPU parity at the full workload sizes, on sampled outputs.

Each test runs the whole path (ab_forward: select -> sample -> attention) on
the full layer, in the launch configuration the benchmark uses, and checks a
sample of (head, query block) rows against the oracle:

* P rows: the GPU's block-mass estimate against the oracle's (independent
  centroids), relative L2 below 2e-2;
* selection: the oracle's SIP on the oracle's own P agrees with the GPU's
  lists on >= 99.5% of kept blocks;
* sampler: the oracle's SIP on the GPU's P rows is bit-exact with the GPU's
  idx / pi_q32 / count;
* attention: the oracle's reweighted attention on the GPU's lists, within
  max-abs 2e-2 (+ bf16 output rounding) and relative L2 5e-3.

Workloads: Wan2.1-480p (B=1, H=40, 21x30x52 tokens), HunyuanVideo-720p
(H=24, 33x45x80 tokens; oracle on 2 heads x 16 query blocks) and the Wan-720p
sweep (H=40, 21x45x80 tokens; KV block x keep ratio x C, and C = 1, the
mean-query proxy), dense attention at the Wan-720p shape, and cross-attention
of the Wan2.1-480p clip to a 9-frame reference clip (14040 keys).
"""
import numpy as np
import pytest

import oracle
from helpers import assert_close_attention, rel_l2, selection_agreement

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_sparse_attention_queries_b200 as ab  # noqa: E402
from block_sparse_attention_queries_b200.synthetic import WORKLOADS, make_workload_qkv  # noqa: E402


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from block_sparse_attention_queries_b200 import build as abbuild
    abbuild.build()
    ab.lib()
    return torch.device("cuda:0")


_QKV = {}


def _workload_inputs(name, dev):
    """Host bf16 Q/K/V of a workload (generated once per module) and device copies."""
    if name not in _QKV:
        _QKV.clear()  # hold one full-size workload at a time
        Qc, Kc, Vc = make_workload_qkv(WORKLOADS[name])
        _QKV[name] = ((Qc, Kc, Vc), tuple(t.to(dev) for t in (Qc, Kc, Vc)))
    return _QKV[name]


def _spread(n, k):
    """k query blocks spread over [0, n), always including the first and the last."""
    return sorted(set(int(round(x)) for x in np.linspace(0, n - 1, k)))


def _check_rows(p, host, bufs, heads, qblocks, what):
    Qc, Kc, Vc = host
    Kb = oracle.budget(p.Nkv, p.keep_ratio)
    assert Kb == ab.budget(p)
    qsel = torch.tensor(qblocks, dtype=torch.long)
    units = []
    data = {}
    for h in heads:
        Qn, Kn, Vn = (t[0, h].float().numpy() for t in (Qc, Kc, Vc))
        Pg = bufs.P[0, h].index_select(0, qsel.to(bufs.P.device)).cpu().numpy()
        gi = bufs.idx[0, h].index_select(0, qsel.to(bufs.idx.device)).cpu().numpy()
        gp = bufs.pi_q32[0, h].index_select(0, qsel.to(bufs.idx.device)).cpu().numpy().view(np.uint32)
        gc = bufs.count[0, h].index_select(0, qsel.to(bufs.idx.device)).cpu().numpy()
        Po = oracle.select_head(Qn, Kn, p.q_block, p.kv_block, p.C, p.kmeans_iters, rows=qblocks)
        assert rel_l2(Pg, Po) < 2e-2, (what, h, rel_l2(Pg, Po))
        data[h] = (Qn, Kn, Vn, Pg, Po, gi, gp, gc)
        units += [(h, r) for r in range(len(qblocks))]

    def one(u):
        h, r = u
        Qn, Kn, Vn, Pg, Po, gi, gp, gc = data[h]
        i = qblocks[r]
        c = int(gc[r])
        si, sp, sc = oracle.sip_row(Pg[r], Kb, p.seed, 0, h, i)          # bit-exact target
        oi, _, _ = oracle.sip_row(Po[r].astype(np.float32), Kb, p.seed, 0, h, i)
        O_ref = oracle.ht_attention_block(Qn, Kn, Vn, p.q_block, p.kv_block, i, gi[r], gp[r], c)
        return u, (si, sp, sc, oi, O_ref)

    res = dict(oracle.run_units(one, units))
    pairs = []
    for (h, r), (si, sp, sc, oi, O_ref) in res.items():
        Qn, Kn, Vn, Pg, Po, gi, gp, gc = data[h]
        c = int(gc[r])
        assert c == sc, (what, h, qblocks[r], c, sc)
        np.testing.assert_array_equal(gi[r][:c], si)
        np.testing.assert_array_equal(gp[r][:c], sp)
        pairs.append((gi[r][:c], oi))
        i = qblocks[r]
        n_i = O_ref.shape[0]
        O_gpu = bufs.O[0, h, i * p.q_block: i * p.q_block + n_i].float().cpu().numpy()
        assert_close_attention(O_gpu, O_ref, f"{what} h={h} i={i}")
    selection_agreement(pairs, what)
    # the whole layer keeps close to the target fraction
    kept = bufs.count.double().mean().item() / p.Nkv
    assert abs(kept - p.keep_ratio) < 0.25 * p.keep_ratio + 2.0 / p.Nkv, (what, kept)


def test_wan480_full_layer(dev):
    w = WORKLOADS["wan480"]
    p = ab.Params.of(w)
    host, (Q, K, V) = _workload_inputs("wan480", dev)
    bufs = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    assert ab.device_error(dev) == 0
    _check_rows(p, host, bufs, heads=[0, 13, 26, 39], qblocks=_spread(p.Nq, 4), what="wan480")


def test_hunyuan720_two_heads_sixteen_blocks(dev):
    w = WORKLOADS["hunyuan720"]
    p = ab.Params.of(w)
    host, (Q, K, V) = _workload_inputs("hunyuan720", dev)
    bufs = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    assert ab.device_error(dev) == 0
    _check_rows(p, host, bufs, heads=[0, w.H - 1], qblocks=_spread(p.Nq, 16), what="hunyuan720")


def test_cross_wan480_full_layer(dev):
    # cross-attention at full size: the Wan2.1-480p clip (32760 queries)
    # attending to a 9-frame reference clip (14040 keys)
    w = WORKLOADS["cross_wan480"]
    p = ab.Params.of(w)
    assert p.L_kv == 14040
    host, (Q, K, V) = _workload_inputs("cross_wan480", dev)
    bufs = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    assert ab.device_error(dev) == 0
    _check_rows(p, host, bufs, heads=[0, 21, 39], qblocks=_spread(p.Nq, 4), what="cross_wan480")


@pytest.mark.parametrize("kvb", [16, 32, 64])
@pytest.mark.parametrize("keep", [0.05, 0.10, 0.20])
@pytest.mark.parametrize("C", [4, 8, 16])
def test_wan720_sweep(dev, kvb, keep, C):
    w = WORKLOADS["wan720"].with_(kv_block=kvb, keep_ratio=keep, C=C)
    p = ab.Params.of(w)
    host, (Q, K, V) = _workload_inputs("wan720", dev)
    bufs = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    assert ab.device_error(dev) == 0
    _check_rows(p, host, bufs, heads=[0, w.H - 1], qblocks=_spread(p.Nq, 3), what=f"wan720 kvb{kvb} r{keep} C{C}")


@pytest.mark.parametrize("kvb,keep", [(16, 0.10), (64, 0.05)])
def test_wan720_mean_query_proxy(dev, kvb, keep):
    # C = 1: one centroid per query block, the block's mean query, scores every
    # KV block (a selector variant, the coarsest IBCS)
    w = WORKLOADS["wan720"].with_(kv_block=kvb, keep_ratio=keep, C=1)
    p = ab.Params.of(w)
    host, (Q, K, V) = _workload_inputs("wan720", dev)
    bufs = ab.ab_forward(p, Q, K, V)
    torch.cuda.synchronize()
    assert ab.device_error(dev) == 0
    _check_rows(p, host, bufs, heads=[0, w.H - 1], qblocks=_spread(p.Nq, 3), what=f"wan720 C1 kvb{kvb} r{keep}")


def test_wan720_dense_sampled_rows(dev):
    w = WORKLOADS["wan720"]
    p = ab.Params.of(w)
    host, (Q, K, V) = _workload_inputs("wan720", dev)
    O = ab.ab_attention_dense(p, Q, K, V)
    torch.cuda.synchronize()
    assert ab.device_error(dev) == 0
    Qc, Kc, Vc = host
    units = [(h, i) for h in (0, w.H - 1) for i in _spread(p.Nq, 2)]
    cache = {h: tuple(t[0, h].float().numpy() for t in (Qc, Kc, Vc)) for h in (0, w.H - 1)}

    def one(u):
        h, i = u
        Qn, Kn, Vn = cache[h]
        n = min(p.q_block, p.L - i * p.q_block)
        return u, oracle.dense_rows(Qn, Kn, Vn, i * p.q_block, n)

    for (h, i), ref in oracle.run_units(one, units):
        got = O[0, h, i * p.q_block: i * p.q_block + ref.shape[0]].float().cpu().numpy()
        assert_close_attention(got, ref, f"dense wan720 h={h} i={i}")

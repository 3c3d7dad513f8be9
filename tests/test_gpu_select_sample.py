"""ab_select_sample (IBCS scoring with SIP run on the rows just scored) on a
B200: its P and block lists equal those of ab_select followed by ab_sample bit
for bit, and the lists equal the oracle's SIP on the GPU's P (AB-Attention
page, "AB-Attention ve Üç Temel Yeniliği", IBCS and SIP items).  The cases
span rows handled by the fused kernel (at most 2048 KV blocks, the
Wan2.1-480p layer among them) and longer rows, for which the call runs the two
steps back to back."""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import oracle  # noqa: E402
from helpers import oracle_sip_rows  # noqa: E402

torch = pytest.importorskip("torch")

import block_sparse_attention_queries_b200 as ab  # noqa: E402
from block_sparse_attention_queries_b200.synthetic import WORKLOADS, make_workload_qkv  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda:0")


def _compare(p, P0, l0, P1, l1, rows):
    assert torch.equal(P0, P1)
    c0, c1 = l0[2].cpu().numpy(), l1[2].cpu().numpy()
    np.testing.assert_array_equal(c0, c1)
    i0, i1 = l0[0].cpu().numpy(), l1[0].cpu().numpy()
    q0, q1 = l0[1].cpu().numpy(), l1[1].cpu().numpy()
    for r in rows:
        n = int(c0[r])
        np.testing.assert_array_equal(i0[r][:n], i1[r][:n])
        np.testing.assert_array_equal(q0[r][:n], q1[r][:n])


@pytest.mark.parametrize("wname,kw", [
    ("tiny", {}),
    ("small", {}),
    ("small", {"C": 16, "seed": 2**63 + 7}),
    ("small", {"C": 1, "keep_ratio": 1.0}),
    ("cross_short", {}),
    ("cross_long", {}),
    ("wan480", {}),
    ("wan720", {"H": 2}),
])
def test_fused_equals_two_calls(dev, wname, kw):
    seed = kw.pop("seed", 42)
    w = WORKLOADS[wname].with_(**kw)
    p = ab.Params.of(w, seed=seed)
    Qc, Kc, _ = make_workload_qkv(w)
    Q, K = Qc.to(dev), Kc.to(dev)
    ws = ab.alloc_workspace(p, dev)
    P0 = ab.ab_select(p, Q, K, workspace=ws)
    l0 = ab.ab_sample(p, P0)
    # caller-owned outputs filled with junk: the fused call writes every entry it reports
    P1 = torch.full_like(P0, float("nan"))
    l1 = tuple(torch.full_like(t, -7) for t in l0)
    got = ab.ab_select_sample(p, Q, K, workspace=ws, out=(P1,) + l1)
    torch.cuda.synchronize()
    assert ab.device_error(dev) == 0
    assert got[0].data_ptr() == P1.data_ptr()
    units = [(b, h, i) for b in range(p.B) for h in range(p.H) for i in range(p.Nq)]
    _compare(p, P0, l0, P1, l1, units)
    # the oracle's SIP on the GPU's P, on a sample of rows
    Pn = P1.cpu().numpy()
    Kb = oracle.budget(p.Nkv, p.keep_ratio)
    rows = units[:: max(1, len(units) // 48)] + [units[-1]]
    ref = oracle_sip_rows(Pn, Kb, p.seed, rows)
    gi, gp, gc = l1[0].cpu().numpy(), l1[1].cpu().numpy().view(np.uint32), l1[2].cpu().numpy()
    for r in rows:
        oi, op, on = ref[r]
        assert gc[r] == on, r
        np.testing.assert_array_equal(gi[r][:on], oi)
        np.testing.assert_array_equal(gp[r][:on], op)


def test_fused_repeatable_and_seeded(dev):
    # same seed: the same lists on every call; another seed: other draws from the same P
    w = WORKLOADS["small"]
    p = ab.Params.of(w, seed=5)
    Qc, Kc, _ = make_workload_qkv(w)
    Q, K = Qc.to(dev), Kc.to(dev)
    a = ab.ab_select_sample(p, Q, K)
    b = ab.ab_select_sample(p, Q, K)
    q = ab.Params.of(w, seed=6)
    c = ab.ab_select_sample(q, Q, K)
    torch.cuda.synchronize()
    assert ab.device_error(dev) == 0
    assert torch.equal(a[0], b[0]) and torch.equal(a[3], b[3])
    assert torch.equal(a[0], c[0])
    assert not torch.equal(a[1], c[1])

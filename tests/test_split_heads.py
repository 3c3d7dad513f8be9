"""A layer's heads divided among ranks (no data collective), on CPU with two
gloo ranks and the CPU oracle.

Every (b, h) is independent on the whole path, so each rank runs
ab_forward_slice on a contiguous slice of the flattened B * H heads.  What the
partition must get right is covered here without a GPU:

* head_slices: the slices are contiguous, disjoint, cover every head, and
  differ in size by at most one head;
* slice_rows: a slice's rows carry the whole problem's (b, h, i) counters, so
  SIP run by each rank on its own rows, with those counters, gives exactly the
  lists of one rank running the whole layer (bit for bit, oracle SIP).

The library's own use of the counters (ab_forward_slice against ab_forward on
one GPU) is checked by tests/test_gpu_parity.py::test_forward_slices_equal_forward."""
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path.insert(0, ROOT)

import block_sparse_attention_queries_b200 as ab  # noqa: E402
import oracle  # noqa: E402

P_SHAPE = dict(B=2, H=3, L=640, d=64, q_block=128, kv_block=16, keep_ratio=0.2, seed=9)  # Nq 5, Nkv 40


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _block_mass(p):
    rng = np.random.default_rng(31)
    x = rng.standard_normal((p.B, p.H, p.Nq, p.Nkv)) * 2.5
    P = np.exp(x - x.max(-1, keepdims=True))
    return (P / P.sum(-1, keepdims=True)).astype(np.float32)


def _rank_main(rank, world, port, q):
    import datetime
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        p = ab.Params(**P_SHAPE)
        P = _block_mass(p)
        Kb = oracle.budget(p.Nkv, p.keep_ratio)
        bh0, nbh = ab.head_slices(p.B, p.H, world)[rank]
        lists = []
        for (b, h, i) in ab.slice_rows(p, bh0, nbh):
            idx, pq, n = oracle.sip_row(P[b, h, i], Kb, p.seed, b, h, i)
            lists.append((np.asarray(idx[:n]).tolist(), np.asarray(pq[:n]).tolist()))
        got = [None] * world
        dist.all_gather_object(got, (rank, bh0, nbh, lists))  # collected for the check only
        if rank == 0:
            q.put(got)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_reproduce_the_single_rank_lists():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    got = q.get(timeout=180)
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    p = ab.Params(**P_SHAPE)
    P = _block_mass(p)
    Kb = oracle.budget(p.Nkv, p.keep_ratio)
    # one rank, the whole layer, rows in [B, H, Nq] order
    full = []
    for b in range(p.B):
        for h in range(p.H):
            for i in range(p.Nq):
                idx, pq, n = oracle.sip_row(P[b, h, i], Kb, p.seed, b, h, i)
                full.append((np.asarray(idx[:n]).tolist(), np.asarray(pq[:n]).tolist()))
    heads = []
    joined = []
    for r, (rank, bh0, nbh, lists) in enumerate(sorted(got)):
        assert rank == r and len(lists) == nbh * p.Nq
        heads.extend(range(bh0, bh0 + nbh))
        joined.extend(lists)
    assert heads == list(range(p.B * p.H))   # contiguous, disjoint, complete, in rank order
    assert joined == full                     # bit for bit


def test_head_slices_partition():
    for B, H in ((1, 40), (1, 24), (2, 3), (3, 5)):
        n = B * H
        for world in range(1, min(n, 9) + 1):
            s = ab.head_slices(B, H, world)
            assert len(s) == world and s[0][0] == 0
            assert all(a0 + an == b0 for (a0, an), (b0, _) in zip(s, s[1:]))
            assert sum(nbh for _, nbh in s) == n
            assert max(nbh for _, nbh in s) - min(nbh for _, nbh in s) <= 1
    with pytest.raises(ValueError):
        ab.head_slices(1, 2, 3)


def test_slice_rows_are_the_whole_problems_rows():
    p = ab.Params(**P_SHAPE)
    rows = [(b, h, i) for b in range(p.B) for h in range(p.H) for i in range(p.Nq)]
    for world in (1, 2, 4, 6):
        joined = []
        for bh0, nbh in ab.head_slices(p.B, p.H, world):
            joined.extend(ab.slice_rows(p, bh0, nbh))
        assert joined == rows

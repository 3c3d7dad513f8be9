"""The multi-rank host logic of bench.py on CPU: two gloo ranks.

One process per GPU, weak scaling: each rank runs its own layer (seeded per
rank), the step time is the maximum over ranks, the value is the whole job's
(world x one layer per step), the reference arm runs on rank 0 only.  The
CUDA path itself is not exercised here."""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, wsz, local = bench.dist_env(world)
        seed = bench.rank_data_seed(r)
        ms = bench.max_over_ranks(10.0 + 5.0 * r, wsz)   # rank 1 is the slow one
        w = bench.workload(type("A", (), {"workload": "wan480"})())
        value = bench.whole_job_value(w, wsz, ms)
        ref = bench.run_reference(type("A", (), {"gpus": world})()) if r != 0 else "skipped"
        q.put((r, wsz, local, seed, ms, value, ref))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = bench.workload(type("A", (), {"workload": "wan480"})())
    seeds = set()
    for r, (rank, wsz, local, seed, ms, value, ref) in enumerate(out):
        assert (rank, wsz, local) == (r, world, r)
        assert ms == 15.0                                     # max over ranks on every rank
        assert value == pytest.approx(2 * bench.dense_flop(w) / 15e-3 / 1e12)
        seeds.add(seed)
        if rank != 0:
            assert ref is None                                # reference arm: rank 0 only
    assert len(seeds) == world                                # a different layer per rank


def test_dist_env_checks(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "4")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.dist_env(4) == (1, 4, 1)
    with pytest.raises(SystemExit):
        bench.dist_env(2)                                     # --gpus must match WORLD_SIZE
    monkeypatch.setenv("RANK", "4")
    with pytest.raises(SystemExit):
        bench.dist_env(4)
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    assert bench.max_over_ranks(3.5, 1) == 3.5

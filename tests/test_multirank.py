"""The replica (weak-scaling) plumbing of bench.py across two gloo ranks on CPU:
rank discovery, the max-over-ranks time and the whole-job throughput."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench.rank_env()
        ms = 10.0 + 5.0 * rank           # the slower rank defines the job time
        worst = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        q.put((r, w, lr, worst, bench.whole_job_tops(10**12, 4, w, worst)))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for r, (rank, world, local, worst, tops) in enumerate(got):
        assert (rank, world, local) == (r, 2, r)
        assert worst == 15.0                       # max over ranks, not the local time
        assert tops == pytest.approx(10**12 * 4 * 2 / 15e-3 / 1e12)


def test_single_process_defaults(monkeypatch):
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.rank_env() == (1, 0, 0)
    assert bench.max_over_ranks(3.5, None, None) == 3.5

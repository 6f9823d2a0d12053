"""The N > 1 host logic of bench.py on CPU: two gloo ranks run replicas,
the job's step time is the slowest rank's and the throughput sums the ranks'
work over it.  The path itself has no collective (replicas only)."""
from __future__ import annotations

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


def _worker(rank: int, world: int, port: int, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        # rank r takes (r + 1) ms per step and does 10 * (r + 1) units per step
        per_step_s = (rank + 1) * 1e-3
        units = 10.0 * (rank + 1)
        mx, job = bench.combine_ranks(per_step_s, units, torch.device("cpu"), True)
        q.put((rank, mx, job))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_replicas_take_max_time_and_sum_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for _, mx, job in res:
        assert mx == pytest.approx(2e-3)
        assert job == pytest.approx((10.0 + 20.0) / 2e-3)


def test_single_rank_is_identity():
    import bench

    mx, job = bench.combine_ranks(4e-3, 8.0, torch.device("cpu"), False)
    assert mx == 4e-3 and job == pytest.approx(2000.0)

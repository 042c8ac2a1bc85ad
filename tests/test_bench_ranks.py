"""bench.py's multi-rank plumbing on CPU: two gloo ranks, each timing its own
replica; the reported time is the max over ranks and the work the sum."""
from __future__ import annotations

import os
import socket

import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [1.5, 4.0][rank]  # this rank's step time
        units = [100.0, 300.0][rank]  # this rank's bytes
        q.put((rank, bench.max_over_ranks(ms, world), bench.sum_over_ranks(units, world)))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_summed_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, total in got:
        assert mx == 4.0 and total == 400.0


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(2.5, 1) == 2.5
    assert bench.sum_over_ranks(7.0, 1) == 7.0

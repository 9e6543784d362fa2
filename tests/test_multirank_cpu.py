"""The N>1 bench path on CPU: two gloo ranks, each with its own problem; the job
time is the slowest rank's and the value counts every rank's tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 * (rank + 1), dist, "cpu")
        dist.barrier()
        q.put((rank, ms, bench.job_throughput(world, 1 << 20, ms)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_and_count_all_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, value in got:
        assert ms == 20.0
        assert value == pytest.approx(2 * (1 << 20) / 0.020 / 1e6)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(1, 1000, 1.0) == pytest.approx(1.0)

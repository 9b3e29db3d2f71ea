"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2): every rank
runs an independent replica (the verification step shards by sequence with no
exchange), the job time is the maximum over ranks, and the value counts the
work of all ranks."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        local_ms = 10.0 + 5.0 * rank  # the slower rank decides the job time
        ms = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value = bench.whole_job_rate(world, units_per_rank=64, ms_total_max=ms, steps=10)
        bench.barrier(world)
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_max_time_and_whole_job_value():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(100)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in res:
        assert ms == 15.0  # max over ranks
        assert value == pytest.approx(2 * 64 / (15.0 / 10 * 1e-3))


def test_single_rank_is_plain():
    import bench

    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert bench.whole_job_rate(1, 64, 20.0, 10) == pytest.approx(64 / 2e-3)

"""The multi-GPU bench logic on CPU: two gloo ranks, max-over-ranks timing and the job value."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local = [80.0, 95.5][rank]                 # each rank's own step time
        m = bench.max_over_ranks_on(local, "cpu", world)
        q.put((rank, m, bench.job_ms_per_layer(m, 1, world)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_take_the_max_and_divide_by_layers():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 95.5, 47.75), (1, 95.5, 47.75)]


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks_on(12.5, "cpu", 1) == 12.5
    assert bench.job_ms_per_layer(12.5, 1, 1) == 12.5

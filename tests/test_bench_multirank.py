"""The benchmark's multi-rank bookkeeping on CPU: two gloo ranks stand in for
two GPUs (each runs its own replica, the slowest rank's time counts)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, local_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        value, ms = bench.job_throughput(world, 32768, local_ms[rank])
        mx = bench.max_over_ranks(local_ms[rank] * 2, world)
        bench.barrier(world)
        out[rank] = (value, ms, mx)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_job_throughput_takes_the_slowest_rank(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    local_ms = [10.0, 12.5]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, local_ms, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(world):
        value, ms, mx = out[r]
        assert ms == 12.5 and mx == 25.0
        assert value == pytest.approx(world * 32768 / 12.5e-3)


def test_single_rank_needs_no_process_group():
    import bench
    value, ms = bench.job_throughput(1, 100, 4.0)
    assert ms == 4.0 and value == pytest.approx(100 / 4e-3)

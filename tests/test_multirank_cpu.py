"""The N > 1 bench path on CPU: two gloo ranks, max-over-ranks timing and the job rate.

The attention path shards into independent replicas with no data-path collective, so the
only cross-rank steps are the timing barrier and the max all-reduce of elapsed time.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    bench.barrier(world)
    m = bench.max_over_ranks(10.0 + rank, world)
    rate = bench.job_throughput(100.0, 5, m, world)
    bench.barrier(world)
    dist.destroy_process_group()
    q.put((rank, m, rate))


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_job_rate(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(world))
    for rank, m, rate in res:
        assert m == 10.0 + world - 1  # the slowest rank's time
        assert rate == pytest.approx(world * 100.0 * 5 / ((10.0 + world - 1) * 1e-3))

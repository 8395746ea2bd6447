"""The N > 1 bench path on CPU: replicas with no data-path collective.

The forward pass shards over independent images, so each rank runs its own
replica; the only cross-rank steps are the barrier around the timed region and
the max over ranks of the step time.  This runs those steps with the gloo
backend, world size 2, on the host.
"""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    my_ms = 10.0 + 5.0 * rank               # rank 1 is the slower replica
    ms = bench.reduce_max(my_ms, world, "cpu")
    flops_per_replica = 1e12
    value = world * flops_per_replica / (ms * 1e-3) / 1e12
    bench.barrier(world)
    dist.destroy_process_group()
    q.put((rank, ms, value))


def test_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]
    assert all(abs(r[2] - 2 * 1e12 / 15e-3 / 1e12) < 1e-9 for r in res)

"""World-size-2 host logic of the multi-GPU benchmark path, on CPU (gloo).

Each rank runs its own replica of the workload (documents are independent,
so there is no data-path collective); the job's time is the maximum of the
ranks' device-timed totals and the job's units are the sum over ranks.
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(10.0 + rank * 5.0, world)  # rank 1 is the slowest
        units = bench.job_tokens(4096, world)
        q.put((rank, t, units))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_timing_and_units():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(world))
    assert [r[1] for r in res] == [15.0, 15.0]
    assert [r[2] for r in res] == [8192, 8192]

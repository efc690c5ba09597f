"""Host-side logic of the multi-rank bench on CPU: two gloo ranks take the
same collective steps (barrier, max over ranks of the elapsed time) as the
NCCL ranks of `bench.py --gpus N`, and a rank that fails is reported as an
error by the others through the process-group timeout, not a hang."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        bench.barrier(world)
        # each rank "measured" a different time; everyone must see the max
        t = bench.allreduce_max(10.0 + rank, world, torch.device("cpu"))
        q.put((rank, t))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_barrier_and_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(60)
    assert all(p.exitcode == 0 for p in ps)
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert got == [(0, 11.0), (1, 11.0)]


def _failing_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        os._exit(3)                      # this rank dies between steps
    try:
        t = torch.tensor([1.0])
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        q.put("no error")
    except Exception as e:               # the survivor learns of it, with an error
        q.put(type(e).__name__)


def test_dead_rank_surfaces_as_error_not_hang():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_failing_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(90)
    assert ps[1].exitcode == 3
    assert q.get(timeout=5) != "no error"

"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (spawned
processes, rendezvous on 127.0.0.1) pass the barrier, agree on the slowest
rank's time, and only rank 0 runs the reference arm."""

import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    slowest = bench.max_over_ranks(10.0 + 5.0 * rank, world)     # rank r took 10 + 5r ms
    ref = bench.run_reference(None, rank, world) if rank != 0 else "rank 0 runs it"
    bench.barrier(world)
    dist.destroy_process_group()
    out.put((rank, slowest, ref))


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict((r, (t, ref)) for r, t, ref in (out.get(timeout=5) for _ in range(world)))
    assert got[0][0] == got[1][0] == 15.0                  # max over ranks, on every rank
    assert got[1][1] is None                               # the reference arm: rank 0 alone

"""The N > 1 bench path on CPU: two gloo ranks join the group the way torchrun
describes it, hit the barrier, and agree on the slowest rank's time; the
whole-job rate counts the units of every rank over that time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup("gloo")
    bench.barrier(w)
    my_ms = 100.0 + 50.0 * r           # rank 1 is the slow one
    m = bench.max_over_ranks(my_ms, w, device="cpu")
    rate = bench.job_throughput(10.0, 4, w, m)
    q.put((r, w, m, rate))
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for r, w, m, rate in got:
        assert w == 2 and m == 150.0
        assert rate == pytest.approx(2 * 10.0 * 4 / 0.150)

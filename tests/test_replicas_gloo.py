"""The multi-process path of bench.py (one replica per rank; ranks meet only
for the timing barrier and the max over ranks), run as two gloo ranks on the
CPU."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    D = bench.Dist(backend="gloo")
    D.barrier()
    m = D.max(10.0 + rank)          # each rank's device time; the job takes the slowest
    D.barrier()
    q.put((rank, m, D.world))
    D.close()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in ps)
    assert got == [(0, 11.0, 2), (1, 11.0, 2)]


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    D = bench.Dist()
    assert D.world == 1 and not D.pg and D.max(3.5) == 3.5

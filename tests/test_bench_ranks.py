"""Replica timing of bench.py on CPU: two gloo ranks report different step
times; the job's time is the slowest rank's and the throughput aggregates
every rank's tokens over it."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    r, w, local, pg = bench.dist_setup()
    try:
        assert (r, w) == (rank, world) and pg.get_backend() == "gloo"
        mine = [1.5, 2.25][rank]
        bench.barrier(pg)
        slow = bench.max_over_ranks(pg, mine)
        q.put((rank, slow, bench.aggregate_throughput(256 * 5, w, slow)))
    finally:
        pg.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slow, thr in res:
        assert slow == 2.25
        assert thr == pytest.approx(256 * 5 * 2 / 2.25)

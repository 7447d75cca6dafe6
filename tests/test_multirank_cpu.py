"""The multi-GPU bench path on CPU: world size 2 over gloo (127.0.0.1).

N replicas run independent copies of the operator (no data-path collective);
the only exchange is the max over ranks of the timed total, from which the
whole-job edges/s is formed. This checks that reduction with unequal rank
times, on two real processes.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    import datetime
    import sys

    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = 10.0 * (rank + 1)                  # rank 0: 10 ms, rank 1: 20 ms
        q.put((rank, bench.aggregate_ranks(t, 1000, 5, world, dist, "cpu")))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        t, v = out[r]
        assert t == pytest.approx(20.0)                       # the slower rank's time
        assert v == pytest.approx(1000 * 2 * 5 / 20e-3)        # edges of both ranks / max time


def test_single_rank_no_collective():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    t, v = bench.aggregate_ranks(8.0, 500, 4, 1)
    assert t == 8.0 and v == pytest.approx(500 * 4 / 8e-3)

"""bench.py's multi-rank host logic on two CPU processes (gloo): every rank
gets the slowest rank's time, ranks draw distinct layers, and the whole-job
rate counts every rank's layer over that time.  No GPU involved."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import sys
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(10.0 + 3.0 * rank, dist, "cpu")
        q.put((rank, t, bench.rank_seed(2, rank)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_share_the_max_time_and_draw_distinct_layers():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [13.0, 13.0]      # both ranks see the slower time
    assert got[0][2] != got[1][2]                   # distinct seeds, distinct layers


def test_single_process_and_rate():
    import bench
    assert bench.max_over_ranks(4.5, None, "cpu") == 4.5
    assert bench.job_rate(2, 4096, 4096, 8.0) == pytest.approx(2 * 4096 * 4096 / 0.008)

"""bench.py's aggregation over ranks, run as two gloo ranks on CPU: every rank reports its own
device time, all of them continue with the slowest one, and the whole-job rate counts every
rank's parameters over that time."""
import os
import socket
from datetime import timedelta

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        ms = bench.max_over_ranks(10.0 * (rank + 1), torch.device("cpu"), world)
        q.put((rank, ms, bench.whole_job_rate(1000, 5, world, ms)))
    finally:
        dist.destroy_process_group()


def test_slowest_rank_time_and_whole_job_rate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert [r[0] for r in results] == [0, 1]
    assert [r[1] for r in results] == [20.0, 20.0]  # rank 1's 20 ms, seen by both ranks
    assert all(r[2] == 1000 * 5 * 2 / 0.020 for r in results)


def test_single_rank_needs_no_process_group():
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks(12.5, torch.device("cpu"), 1) == 12.5
    assert bench.whole_job_rate(6_738_415_616, 100, 1, 2000.0) == 6_738_415_616 * 100 / 2.0
